// minikv_decode_attn: one decoding step over the 2-bit cache (flash-decoding).
//
// Source: MiniKV abstract (specialized CUDA kernels compatible with
// FlashAttention) and the gptget.net summary of arXiv 2411.18077, section
// 方法论 (sub-channel key / per-token value 2-bit quantization, compact layout).
//
// Work list.  Every (sequence, KV head) "unit" contributes, in order,
//   * residual items: 5 fp16 residual tokens each (the new token included), and
//   * packed items:   32 packed tokens each (one slice of one key group).
// The items of all units are laid end to end and cut, by weight (packed 8,
// residual 7: their measured costs; plus a boundary weight before each unit,
// picked per call by a cost model of the slowest CTA, see the host partition
// below), into one contiguous range per SM.  One CTA of 16 warps runs on each
// SM that takes a range.  Its warps claim the items of its range one
// at a time from a shared-memory counter (so warps the scheduler favours simply
// take more items, and all finish together) and stream them through per-warp
// 3-stage cp.async pipelines (16 bytes per lane per copy, written to
// bank-conflict-free positions).  Each warp keeps an online-softmax state per
// query head.  At the end of each unit the 16 warps merge their states in
// shared memory and the CTA writes one partial (m, l, sum p*v) per head; the
// last CTA to arrive at a unit (self-resetting atomic counter) merges the
// unit's partials into `out`, and when the residual ring is full it also packs
// the oldest G residual tokens into a new key group.
//
// Packed-item math (per warp, 32 tokens = 2 m-tiles of 16, g <= 4 heads):
//   codes -> fp16 SUBNORMALS: one AND puts a 2-bit code at mantissa bit p of
//     both halves of a 32-bit word (value code * 2^(p-24); the tensor cores
//     take fp16 subnormals exactly);
//   scores S[tok, n] = sum_c code_c 2^(p_c-24) b_c over mma.sync.m16n8k16, with
//     the 8 B columns interleaved per head: column 2h holds the fp16 "hi" part
//     of q_h,c s_c 2^-p_c, column 2h+1 the exact remainder ("lo"), so the lane
//     that owns head h holds both parts of its score (no shuffle) and every
//     (token, head) probability is computed once;
//   the key zero-point term sum_c q_c z_c takes two mma: A rows are (head,
//     16-channel chunk) of q, B columns are chunks of the zero row, and the
//     term of a head is the sum of four diagonal entries (two shuffles);
//   output O^T[ch, n] = sum_t code_{t,ch} 2^(p-24) P'[t, n], P' = p_t v_scale_t
//     split hi / lo the same way and moved into the B layout by movmatrix;
//     out_ch = (O^T[ch, 2h] + O^T[ch, 2h+1]) 2^(24-p) + sum_t p_t v_zero_t.
// Residual items use the fp16 rows directly: K through ldmatrix, V through
// 128-bit loads arranged into the same accumulator layout as packed values.
//
// Attention-mass variant (minikv_decode_attn_mass): every warp also stores the
// absolute log2 score of each token it scores, per query head; the merging
// CTA of a unit stores the unit's final (max, sum) per head; mass_kernel then
// adds sum_h 2^(x_h,t - M_h) / L_h to the caller's running score of token t,
// the H2O-style accumulated attention the MiniKV summary's experiments compare
// with.
#include <math.h>

#include <atomic>
#include <map>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace minikv {

namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kSlice = 32;           // packed tokens per packed item
constexpr int kResTok = 5;           // residual tokens per residual item
constexpr int kStages = 3;           // per-warp pipeline depth
constexpr int kStageBytes = 2688;    // one packed item (a residual item takes 2560)
constexpr int kWP = 8, kWR = 7;      // partition weights of a packed / residual item (measured cost ratio)
constexpr int kWU = 640;             // partition weight of a unit boundary in the device-state mode (the
                                     // host-planned modes pick one per call); also the floor of min_share
constexpr int kMinShare = kWU + 8 * kWP;   // least weight per CTA at the default boundary weight
// least weight per CTA for boundary weight wu: a range always holds an item
// start, and never less than at the default weight (the partial slots of the
// workspace are sized for that share)
constexpr long long min_share(int wu) { return (long long)(wu > kWU ? wu : kWU) + 8 * kWP; }
constexpr int kPartStride = 132;     // floats per (unit, slot, head): y[128], m, l
constexpr int kMaxCtas = 512;
constexpr float kLazy = 8.f;         // log2 headroom before a head's reference max moves
constexpr int kWyStride = kD + 4;    // floats per (warp, head) row of the warp states

// packed stage: K codes [32 rows x 32 B] (rows permuted by kpos), V codes the
// same, k_scale / k_zero 16 chunks each (permuted by schunk), v_scale, v_zero
constexpr int kOffKc = 0, kOffVc = 1024, kOffKs = 2048, kOffKz = 2304, kOffVs = 2560, kOffVz = 2624;
// residual stage: K rows [5][256 B] (chunks XOR-swizzled by row), V rows (chunks rotated by rvrot)
constexpr int kOffRk = 0, kOffRv = kResTok * 256;
static_assert(2 * kResTok * 256 <= kStageBytes, "residual item fits a stage");

// One unit's share of a CTA's range ("segment").
struct Seg {
    int u, b, ub, items, nri, nq, r, rs, first, S_u, hi;
};

struct __align__(16) Smem {
    unsigned char stage[kWarps][kStages][kStageBytes];
    unsigned char qbuf[kWarps][kStages][4 * 256];   // query rows of a unit: [head][16 chunks], chunk c at c ^ head
    float wm[kWarps][4], wl[kWarps][4];
    float wy[kWarps][4][kWyStride];                 // per warp and head; padded: conflict-free 16-byte stores
    uint4 zero;
    int flag;
    int next;   // next item of the CTA's range to claim
    Seg seg;    // the unit being processed
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
    unsigned *grid_counter;   // device-state mode: CTAs of this launch that have finished (self-resetting)
    int *dseq;                // device-state mode: per-sequence state [B][4] in device memory
    float *xs;                // mass variant: absolute log2 scores [unit][g][xs_stride]
    float *stats;             // mass variant: per unit max[4], sum[4], token count (int bits), pad
    int xs_stride;
    int Hkv, g, G, cap, ring;
    int n_q, r, res_start;    // uniform batch: every sequence's lengths (r counts the new token)
    int det;                  // 1: items go to warps round robin (no claiming): a fixed schedule
    int units, P, S_max;      // CTAs that take a share, partial slots per unit
    int nb;                   // sequences (units / Hkv)
    int groups_cap, lg2G;     // cap / G and log2(G)
    float scale_log2;
};

// Host-planned modes: the first flat item of each CTA's range (P + 1 entries).
struct CtaTab {
    int lo[kMaxCtas + 1];
};

// ---- per-unit item counts
__host__ __device__ __forceinline__ int unit_nri(int r) { return (r + kResTok - 1) / kResTok; }
__host__ __device__ __forceinline__ int unit_items(int nq, int r) { return unit_nri(r) + nq / kSlice; }
// a unit's weight: its boundary (weight wu), then its items
__host__ __device__ __forceinline__ long long unit_w(int nq, int r, int wu = kWU) {
    return wu + (long long)unit_nri(r) * kWR + (long long)(nq / kSlice) * kWP;
}
// the item of a unit (nri residual items) whose start weight is the first one
// at or after `rem` (0 <= rem < the unit's weight)
__host__ __device__ __forceinline__ int item_at(long long rem, int nri, int wu = kWU) {
    rem = rem > wu ? rem - wu : 0;
    if (rem <= (long long)(nri - 1) * kWR) return (int)((rem + kWR - 1) / kWR);
    return nri + (int)((rem - (long long)nri * kWR + kWP - 1) / kWP);
}

// ---- sequence lengths and item prefix sums, by mode.  Uniform batches read the
// shared scalars; ragged ones a kernel-parameter table; device-state ones a
// table each CTA builds in shared memory from the device-resident state.
struct ArgsUni : Args {
    CtaTab cta;
};
__host__ __device__ __forceinline__ int nseq(const Args &a) { return a.nb; }
__device__ __forceinline__ int s_nq(const ArgsUni &a, int) { return a.n_q; }
__device__ __forceinline__ int s_r(const ArgsUni &a, int) { return a.r; }
__device__ __forceinline__ int s_rs(const ArgsUni &a, int) { return a.res_start; }
__device__ __forceinline__ int s_ibeg(const ArgsUni &a, int b) { return b * a.Hkv * unit_items(a.n_q, a.r); }
__device__ __forceinline__ int seq_of_x(const ArgsUni &a, int x) { return x / (a.Hkv * unit_items(a.n_q, a.r)); }
__device__ __forceinline__ int cta_lo(const ArgsUni &a, int c) { return a.cta.lo[c]; }
__device__ __forceinline__ int part_P(const ArgsUni &a) { return a.P; }

constexpr int kMaxRaggedSeqs = MINIKV_MAX_RAGGED_SEQS;
struct SeqTab {
    int n_q[kMaxRaggedSeqs];
    int r[kMaxRaggedSeqs];
    int res_start[kMaxRaggedSeqs];
    int ibeg[kMaxRaggedSeqs + 1];   // first flat item of sequence b's units
};
struct ArgsVar : Args {
    SeqTab tab;
    CtaTab cta;
};
// largest b with beg(b) <= v (beg(0) = 0 <= v < beg(n))
template <class F>
__device__ __forceinline__ int seq_search(int n, int v, F beg) {
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (beg(mid) <= v) lo = mid;
        else hi = mid;
    }
    return lo;
}
__device__ __forceinline__ int s_nq(const ArgsVar &a, int b) { return a.tab.n_q[b]; }
__device__ __forceinline__ int s_r(const ArgsVar &a, int b) { return a.tab.r[b]; }
__device__ __forceinline__ int s_rs(const ArgsVar &a, int b) { return a.tab.res_start[b]; }
__device__ __forceinline__ int s_ibeg(const ArgsVar &a, int b) { return a.tab.ibeg[b]; }
__device__ __forceinline__ int seq_of_x(const ArgsVar &a, int x) {
    return seq_search(nseq(a), x, [&](int b) { return a.tab.ibeg[b]; });
}
__device__ __forceinline__ int cta_lo(const ArgsVar &a, int c) { return a.cta.lo[c]; }
__device__ __forceinline__ int part_P(const ArgsVar &a) { return a.P; }

// Device-state mode: the table sits behind Smem in dynamic shared memory:
// DevTab, then n_q[B], r[B], res_start[B], ibeg[B + 1], cta_lo[P + 1],
// status[B] (int; P = the launch's partition bound a.P).
struct ArgsDev : Args {};
struct DevTab {
    long long Wt;
    int P;
    int pad;
};
__device__ __forceinline__ unsigned char *dyn_smem() {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    return smem_raw;
}
__device__ __forceinline__ DevTab &dev_tab() { return *reinterpret_cast<DevTab *>(dyn_smem() + sizeof(Smem)); }
__device__ __forceinline__ int *dev_arr(const Args &a, int k) {   // k = 0 n_q, 1 r, 2 res_start, 3 ibeg, 4 cta_lo
    return reinterpret_cast<int *>(dyn_smem() + sizeof(Smem) + sizeof(DevTab)) + k * nseq(a) + (k > 3 ? 1 : 0);
}
__device__ __forceinline__ int s_nq(const ArgsDev &a, int b) { return dev_arr(a, 0)[b]; }
__device__ __forceinline__ int s_r(const ArgsDev &a, int b) { return dev_arr(a, 1)[b]; }
__device__ __forceinline__ int s_rs(const ArgsDev &a, int b) { return dev_arr(a, 2)[b]; }
__device__ __forceinline__ int s_ibeg(const ArgsDev &a, int b) { return dev_arr(a, 3)[b]; }
__device__ __forceinline__ int seq_of_x(const ArgsDev &a, int x) {
    const int *ib = dev_arr(a, 3);
    return seq_search(nseq(a), x, [&](int b) { return ib[b]; });
}
__device__ __forceinline__ int cta_lo(const ArgsDev &a, int c) { return dev_arr(a, 4)[c]; }
__device__ __forceinline__ int part_P(const ArgsDev &) { return dev_tab().P; }

// ---- positions in the work list

// Segment info for the unit holding flat item x, in CTA c's range (one
// thread).  The CTAs that hold items of the unit are c's neighbours: walks
// from c over the range table find the first and the last (entries next to
// c's, mostly in the same constant-cache line; every range is non-empty).
template <class A>
__device__ void seg_info(const A &a, int c, int x, int xhi, Seg &s) {
    const int b = seq_of_x(a, x);
    const int nq = s_nq(a, b), r = s_r(a, b);
    const int items = unit_items(nq, r);
    const int kh = (x - s_ibeg(a, b)) / items;
    s.u = b * a.Hkv + kh;
    s.b = b;
    s.ub = s_ibeg(a, b) + kh * items;
    s.items = items;
    s.nri = unit_nri(r);
    s.nq = nq;
    s.r = r;
    s.rs = s_rs(a, b);
    s.hi = min(xhi, s.ub + items);
    // CTAs that write a partial for the unit: those whose ranges hold its items
    const int P = part_P(a), last = s.ub + items - 1;
    int c0 = c, c1 = c;
    while (c0 > 0 && cta_lo(a, c0) > s.ub) --c0;
    while (c1 < P - 1 && cta_lo(a, c1 + 1) <= last) ++c1;
    s.first = c0;
    s.S_u = c1 - c0 + 1;
}

// A warp's place in the work list: unit u (= b Hkv + kh), item k of the unit,
// ub = flat index of the unit's first item.  Moving forward needs no division.
struct Cursor {
    int x, u, b, kh, k, ub, items;
    template <class A>
    __device__ __forceinline__ void set(const A &a, int x_) {
        x = x_;
        b = seq_of_x(a, x);
        items = unit_items(s_nq(a, b), s_r(a, b));
        kh = (x - s_ibeg(a, b)) / items;
        u = b * a.Hkv + kh;
        ub = s_ibeg(a, b) + kh * items;
        k = x - ub;
    }
    template <class A>
    __device__ __forceinline__ void advance_to(const A &a, int x_) {
        k += x_ - x;
        x = x_;
        while (k >= items) {
            k -= items;
            ub += items;
            ++u;
            if (++kh == a.Hkv) {
                kh = 0;
                ++b;
                items = unit_items(s_nq(a, b), s_r(a, b));
            }
        }
    }
};

// ---- small device helpers

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
__device__ __forceinline__ float warp_sum_g(float x) {   // over the lanes of one head (xor 4, 8, 16)
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
// word >> 10 as an integer multiply-high (IMAD.HI), which issues on the FMA
// pipe and leaves the busier integer ALU to the masks
__device__ __forceinline__ uint32_t shr10(uint32_t x) {
    uint32_t y;
    asm("mul.hi.u32 %0, %1, 4194304;\n" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t w4(const uint4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }
// D (16x8 fp32) += A (16x8 fp16, row) * B (8x8 fp16, col):
//   a0 = {(g,2t),(g,2t+1)}, a1 = {(g+8,2t),(g+8,2t+1)}, b = {(2t,g),(2t+1,g)}; D as for m16n8k16
__device__ __forceinline__ void mma1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};\n"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(b));
}
// arrival on a unit / launch counter: release of this CTA's writes (ordered
// before by a block barrier) and acquire of the earlier arrivals' writes
__device__ __forceinline__ unsigned atom_inc_acq_rel(unsigned *p, unsigned lim) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.inc.u32 %0, [%1], %2;\n" : "=r"(old) : "l"(p), "r"(lim) : "memory");
    return old;
}

// Code pair i (i = 0..7) of a 32-bit word of 16 codes -> fp16x2 subnormals
// (code_i, code_{i+8}) at mantissa bit pair_pos(i): pairs 0..4 are masked
// straight out of the word (bits 0, 2, .., 8 of each half), pairs 5..7 out of
// word >> 10 (bits 0, 2, 4).  x = word, y = word >> 10.
template <int I>
__device__ __forceinline__ uint32_t code_pair(uint32_t x, uint32_t y) {
    if constexpr (I < 5) return x & (0x00030003u << (2 * I));
    else return y & (0x00030003u << (2 * (I - 5)));
}
__host__ __device__ constexpr int pair_pos(int i) { return i < 5 ? 2 * i : 2 * (i - 5); }
// 2^-pos (key B operand: q s 2^-pos stays below the fp16 limit whenever q s
// does) and 2^(24 - pos) (value output scale)
__host__ __device__ constexpr float pair_wq(int i) { return 1.f / (float)(1 << pair_pos(i)); }
__host__ __device__ constexpr float pair_wo(int i) { return (float)(1 << (24 - pair_pos(i))); }
constexpr float kScoreUnit = 16777216.f;   // packed scores come out as code q s 2^-24

// row of packed token j (0..31) in a stage's code block: tokens 2m of a
// 16-token tile (and 2m+1) land in distinct bank groups, and so do tokens 4t+o
__host__ __device__ __forceinline__ int kpos(int j) { return 4 * (j >> 2) + ((j + (j >> 2)) & 3); }
// position of 8-channel chunk k (0..15) of the key scale / zero rows
__host__ __device__ __forceinline__ int schunk(int k) { return k ^ ((k & 8) >> 2); }
// rotation of the 16-byte chunks of residual V row j
__host__ __device__ __forceinline__ int rvrot(int j) { return ((j >> 1) & 1) + 4 * ((j >> 2) & 1); }

// ---------------------------------------------------------------- partials

// The CTA's 16 warp states for the segment's unit (already scaled to the CTA's
// per-head max and written to sm.wy / wl / wm) are summed into one partial in
// slot `slot`; the last CTA of the unit to arrive (S_u arrivals) merges the
// partials into `out` and, if the residual ring is full, packs its oldest G
// tokens into key group n_q/G.  A unit within one CTA is written out directly.
// Thread tid handles head tid / 128, channel tid % 128.
template <bool kMass, class A>
__device__ void finish_unit(const A &a, Smem &sm, const Seg &s, int slot) {
    const int tid = threadIdx.x, h = tid >> 7, ch = tid & 127;
    const int unit = s.u;
    const int b = s.b, kvh = unit - s.b * a.Hkv;
    const int Hq = a.Hkv * a.g;
    __syncthreads();   // warp states written
    float M = -INFINITY, L = 0.f, Y = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        M = fmaxf(M, sm.wm[w][h]);
        L += sm.wl[w][h];
        Y += sm.wy[w][h][ch];
    }
    if (s.S_u > 1) {
        float *base = a.part + ((size_t)unit * a.S_max + slot) * 4 * kPartStride + h * kPartStride;
        if (h < a.g) {
            base[ch] = Y;
            if (ch == 0) {
                base[128] = M;
                base[129] = L;
            }
        }
        __syncthreads();
        if (tid == 0) sm.flag = (atom_inc_acq_rel(&a.counters[unit], (unsigned)(s.S_u - 1)) == (unsigned)(s.S_u - 1));
        __syncthreads();
        if (!sm.flag) return;
        // merge the unit's partials: eight slots per round, every load of a
        // round issued before any is used (online rescaling)
        const float *ub = a.part + (size_t)unit * a.S_max * 4 * kPartStride + h * kPartStride;
        M = -INFINITY;
        L = 0.f;
        Y = 0.f;
        if (h < a.g)
            for (int s0 = 0; s0 < s.S_u; s0 += 8) {
                float ms[8], ls[8], ys[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const bool ok = s0 + j < s.S_u;
                    const float *p = ub + (size_t)(s0 + j) * 4 * kPartStride;
                    ms[j] = ok ? __ldcg(p + 128) : -INFINITY;
                    ls[j] = ok ? __ldcg(p + 129) : 0.f;
                    ys[j] = ok ? __ldcg(p + ch) : 0.f;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float m = ms[j], Mn = fmaxf(M, m);
                    const float fo = (M == -INFINITY) ? 0.f : ex2(M - Mn);
                    const float fs = (m == -INFINITY) ? 0.f : ex2(m - Mn);
                    L = fmaf(L, fo, ls[j] * fs);
                    Y = fmaf(Y, fo, ys[j] * fs);
                    M = Mn;
                }
            }
    }
    if (h < a.g) {
        a.out[((size_t)b * Hq + kvh * a.g + h) * kD + ch] = f2h(__fdividef(Y, L));
        if (kMass && ch == 0) {
            a.stats[unit * 12 + h] = M;
            a.stats[unit * 12 + 4 + h] = L;
        }
    }
    if (kMass && tid == 0) a.stats[unit * 12 + 8] = __int_as_float(s.nq + s.r);
    if (s.r == a.ring && s.nq + a.G <= a.cap) {
        // flush: the oldest G residual tokens (all in the ring: the new token was
        // appended before its CTA arrived) become key group nq/G and G value tokens
        const uint16_t *kres = a.k_res + (size_t)unit * a.ring * kD;
        const uint16_t *vres = a.v_res + (size_t)unit * a.ring * kD;
        const int rs = s.rs;
        auto slot_of = [&](int i) { const int t = rs + i; return t >= a.ring ? t - a.ring : t; };
        auto krow = [&](int i, int c) -> const uint16_t * { return kres + (size_t)slot_of(i) * kD + c; };
        auto vrow = [&](int i, int c) -> const uint16_t * { return vres + (size_t)slot_of(i) * kD + c; };
        const size_t tok0 = (size_t)unit * a.cap + s.nq;
        const size_t grow = (size_t)unit * a.groups_cap + s.nq / a.G;
        float *scr = &sm.wy[0][0][0];   // the warp states are summed: free as scratch
        __syncthreads();
        pack_key_group<kThreads>(krow, a.G, a.k_codes_w + tok0 * 8, a.k_scale_w + grow * kD,
                                 a.k_zero_w + grow * kD, scr);
        pack_value_tokens<kThreads>(vrow, a.G, kD, a.v_codes_w + tok0 * 8, a.v_scale_w + tok0, a.v_zero_w + tok0);
    }
}

// ------------------------------------------------------------------ issuing

// Per-lane constants of the copies of a packed item.
struct PackedLane {
    uint32_t row;       // smem offset of this lane's K / V code chunk (token lane/2, half lane%2)
    uint32_t sz_dst;    // smem offset of its key-scale / key-zero chunk
    uint32_t v_dst;     // smem offset of its value scale / zero chunk (lanes 0-7)
    uint32_t sz_src;    // byte offset of that chunk in a scale / zero row
    uint32_t v_src;     // byte offset in the value scale / zero run
};

// Queue the copies of packed item j (tokens 32j..32j+31) of unit u into the
// stage at `st` (shared address).  Every lane copies 16-byte chunks.
template <class A>
__device__ __forceinline__ void issue_packed(const A &a, uint32_t st, int u, int j, int lane, const PackedLane &pl) {
    const size_t tok = (size_t)u * a.cap + (size_t)j * kSlice;
    const char *kc = reinterpret_cast<const char *>(a.k_codes) + tok * 32 + 16 * lane;
    const char *vc = reinterpret_cast<const char *>(a.v_codes) + tok * 32 + 16 * lane;
    cp_async16(st + kOffKc + pl.row, kc, true);
    cp_async16(st + kOffKc + 512 + pl.row, kc + 512, true);
    cp_async16(st + kOffVc + pl.row, vc, true);
    cp_async16(st + kOffVc + 512 + pl.row, vc + 512, true);
    const size_t grow = (size_t)u * a.groups_cap + ((j * kSlice) >> a.lg2G);
    const char *sz = reinterpret_cast<const char *>(lane < 16 ? a.k_scale : a.k_zero) + grow * (kD * 2);
    cp_async16(st + pl.sz_dst, sz + pl.sz_src, true);
    if (lane < 8) {
        const char *vsz = reinterpret_cast<const char *>(lane < 4 ? a.v_scale : a.v_zero) + tok * 2;
        cp_async16(st + pl.v_dst, vsz + pl.v_src, true);
    }
}

// Residual item i of unit u: logical residual tokens 5i .. 5i+4 (those below r;
// the rest are zero-filled).  Lanes 0-15 copy chunk `lane` of each K row,
// lanes 16-31 chunk `lane - 16` of each V row.  Token r-1 is this step's new
// token, read from k_new / v_new.
template <class A>
__device__ __forceinline__ void issue_residual(const A &a, uint32_t st, int u, int i, int r, int rs, int lane) {
    const int part = lane >> 4, c = lane & 15;
    const uint16_t *newrow = (part ? a.v_new : a.k_new) + (size_t)u * kD + 8 * c;
    const uint16_t *ring = (part ? a.v_res : a.k_res) + (size_t)u * a.ring * kD + 8 * c;
    const int t0 = i * kResTok;
    int slot = rs + t0;
    if (slot >= a.ring) slot -= a.ring;
#pragma unroll
    for (int j = 0; j < kResTok; ++j) {
        const int ti = t0 + j;
        const bool ok = ti < r;
        const uint16_t *src = (ti == r - 1 || !ok) ? newrow : ring + (size_t)slot * kD;
        const uint32_t dst = part == 0 ? st + kOffRk + j * 256 + 16 * (c ^ j)
                                       : st + kOffRv + j * 256 + 16 * ((c + rvrot(j)) & 15);
        cp_async16(dst, src, ok);
        if (++slot == a.ring) slot = 0;
    }
}

// Query rows of unit u (heads >= g zero-filled) into a q buffer: chunk c of
// head h at position c ^ h.
template <class A>
__device__ __forceinline__ void issue_q(const A &a, uint32_t qb, int u, int lane) {
    const int b = u / a.Hkv, kh = u - b * a.Hkv;
    const uint16_t *qrow = a.q + ((size_t)b * a.Hkv * a.g + (size_t)kh * a.g) * kD;
#pragma unroll
    for (int e0 = 0; e0 < 64; e0 += 32) {
        const int e = e0 + lane, h = e >> 4, c = e & 15;
        const bool ok = h < a.g;
        cp_async16(qb + (h * 16 + (c ^ h)) * 16, qrow + (ok ? h : 0) * kD + 8 * c, ok);
    }
}

// ------------------------------------------------------------------ the CTA

__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// kWait: the CTA does its parameter-only set-up, then waits for the previous
// kernel on the stream (programmatic dependent launch) before its first global
// read; otherwise the caller has waited already.
template <bool kMass, bool kWait, class A>
__device__ void run_cta(const A &a, Smem &sm, int c) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g_ = lane >> 2, t_ = lane & 3;
    const int xlo = cta_lo(a, c), xhi = cta_lo(a, c + 1);
    const uint32_t st0 = smem_addr(&sm.stage[warp][0][0]);
    const uint32_t qb0 = smem_addr(&sm.qbuf[warp][0][0]);
    const uint32_t zero_addr = smem_addr(&sm.zero);

    // ---- producer: claims items of [xlo, xhi) and queues them kStages - 1 ahead
    PackedLane pl;
    pl.row = kpos(lane >> 1) * 32 + 16 * (lane & 1);
    pl.sz_dst = (lane < 16 ? kOffKs : kOffKz) + 16 * schunk(lane & 15);
    pl.sz_src = 16 * (lane & 15);
    pl.v_dst = (lane < 4 ? kOffVs : kOffVz) + 16 * (lane & 3);
    pl.v_src = 16 * (lane & 3);
    Cursor pc;
    pc.set(a, min(xlo + warp, xhi - 1));
    int pq_unit = -1, pq_slot = -1, pstage = 0, nclaim = 0, nis = 0;
    int xq0 = xhi, xq1 = xhi, xq2 = xhi;   // claimed items in flight, oldest first (xhi = none)
    int pre = 0;   // lane 0: the next dynamic claim, taken one issue ahead so its latency is hidden
    auto issue_next = [&]() {
        int x = 0;
        if (nis < kStages - 1 || a.det) {   // the first items of each warp are fixed; all of them in det mode
            x = xlo + warp + kWarps * nis;
        } else {
            x = __shfl_sync(0xffffffffu, pre, 0);
            if (lane == 0) pre = atomicAdd(&sm.next, 1);
        }
        ++nis;
        if (x < xhi) {
            pc.advance_to(a, x);
            const uint32_t st = st0 + pstage * kStageBytes;
            if (pc.u != pq_unit) {   // first item of a new unit for this warp: bring its query rows too
                pq_unit = pc.u;
                pq_slot = pq_slot == kStages - 1 ? 0 : pq_slot + 1;
                issue_q(a, qb0 + pq_slot * 1024, pc.u, lane);
            }
            const int r = s_r(a, pc.b), nri = unit_nri(r);
            if (pc.k < nri) issue_residual(a, st, pc.u, pc.k, r, s_rs(a, pc.b), lane);
            else issue_packed(a, st, pc.u, pc.k - nri, lane, pl);
        } else {
            x = xhi;
        }
        cp_async_commit();
        pstage = pstage == kStages - 1 ? 0 : pstage + 1;
        if (nclaim == 0) xq0 = x;
        else if (nclaim == 1) xq1 = x;
        else xq2 = x;
        ++nclaim;
    };
    // set-up of the first segment (kernel parameters and shared memory only: it
    // may overlap the previous kernel's tail; the dynamic claims start after the
    // barrier below)
    if (tid == 0) {
        sm.zero = make_uint4(0, 0, 0, 0);
        sm.next = xlo + kWarps * (kStages - 1);   // the first kStages-1 items of each warp are fixed
        seg_info(a, c, xlo, xhi, sm.seg);
    }
    if (kWait) wait_prior_grid();
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) issue_next();
    __syncthreads();
    if (!a.det && lane == 0) pre = atomicAdd(&sm.next, 1);   // the first dynamic claim

    // ---- consumer constants of this lane
    const float sl2 = a.scale_log2, sl2w = a.scale_log2 * kScoreUnit;
    const uint32_t lo_neg = (g_ & 1) ? 0xBC00BC00u : 0u;   // fp16x2 (-1, -1) in lo columns, (0, 0) in hi
    const int hB = g_ >> 1;                                // head of this lane's B column
    const uint32_t kA = kpos(2 * g_) * 32 + 8 * t_, kB = kpos(2 * g_ + 1) * 32 + 8 * t_;
    const uint32_t vo0 = kpos(4 * t_) * 32 + 4 * g_, vo1 = kpos(4 * t_ + 1) * 32 + 4 * g_;
    const uint32_t vo2 = kpos(4 * t_ + 2) * 32 + 4 * g_, vo3 = kpos(4 * t_ + 3) * 32 + 4 * g_;
    // chunks 4t_ + 2 half (+1) of the key scales (channels 16(2t_+half) .. +15): schunk
    // swaps the two halves of lanes t_ >= 2
    const uint32_t ks_h0 = 64 * t_ + 32 * (t_ >> 1), ks_h1 = 64 * t_ + 32 * (1 - (t_ >> 1));
    // ldmatrix rows of the q B operand: matrix m = lane >> 3 (chunk 4jj + m), row n = lane & 7 ->
    // head n/2 for even n, zero for odd n (the lo columns)
    const int qn = lane & 7;
    const bool q_zero = qn & 1;
    const uint32_t q_row_off = ((qn >> 1) * 16 + ((lane >> 3) ^ (qn >> 1))) * 16;
    // key zero-point term: two mma whose A rows are (head, 16-channel chunk) of q and whose
    // B columns are chunks of the zero row; the term of head h is the sum of the four
    // diagonal entries D[4h' + j][j] (h' = h mod 2; heads 2, 3 in rows 8-15).  Matrix
    // m = lane >> 3 of an A load: rows 8 (m & 1) .. +7, channels 8 (m >> 1) .. +7 of each
    // chunk; the B load: chunks (row & 3) + 4 (m >> 1), channel half m & 1.
    uint32_t zq_off, zz_off;
    {
        const int m = lane >> 3, rr = lane & 7;
        const int row = ((m & 1) << 3) + rr, h = row >> 2, c8 = 2 * (row & 3) + (m >> 1);
        zq_off = h * 256 + ((c8 ^ h) << 4);
        const int cz = 2 * ((rr & 3) + 4 * (m >> 1)) + (m & 1);
        zz_off = kOffKz + 16 * schunk(cz);
    }
    const bool z_diag = t_ == ((g_ & 3) >> 1), z_odd = g_ & 1;
    const int z_src = 16 * (t_ & 1);
    // residual K rows: matrices (chunk 2kk rows, zero, chunk 2kk+1 rows, zero)
    const int rk_row = lane & 7, rk_m = lane >> 3;
    const bool rk_live = !(rk_m & 1) && rk_row < kResTok;
    uint32_t qw[8][2];   // per-segment score B base: (q_c 2^-pos, q_{c+8} 2^-pos), head hB

    int cq_unit = -1, cq_slot = -1, cstage = 0;
    for (;;) {
        const Seg sg = sm.seg;
        const int u = sg.u, ub = sg.ub, nri = sg.nri, nq = sg.nq, r = sg.r, rs = sg.rs;

        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
        float m_ref = -INFINITY, l = 0.f, pz = 0.f;
        bool vunit = false;   // acc holds packed-value units (x 2^(pos-24)) once a packed item was seen
        uint32_t qb = 0;      // this segment's q buffer (shared address)

        while (xq0 < sg.hi) {
            const int x = xq0;
            issue_next();
            cp_async_wait<kStages - 1>();
            __syncwarp();
            const uint32_t S = st0 + cstage * kStageBytes;
            if (u != cq_unit) {   // first item of the segment for this warp: its query rows arrived with it
                cq_unit = u;
                cq_slot = cq_slot == kStages - 1 ? 0 : cq_slot + 1;
                qb = qb0 + cq_slot * 1024;
                const uint32_t qh = qb + hB * 256;
                const uint4 qa0 = lds128(qh + ((4 * t_) ^ hB) * 16);
                const uint4 qb0v = lds128(qh + ((4 * t_ + 1) ^ hB) * 16);
                const uint4 qa1 = lds128(qh + ((4 * t_ + 2) ^ hB) * 16);
                const uint4 qb1v = lds128(qh + ((4 * t_ + 3) ^ hB) * 16);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int half = kk >> 2, Q = kk & 3;
                    const uint32_t wa = w4(half ? qa1 : qa0, Q), wb = w4(half ? qb1v : qb0v, Q);
                    const float w0 = pair_wq(2 * Q), w1 = pair_wq(2 * Q + 1);
                    const __half2 s0 = __floats2half2_rn(w0, w0), s1 = __floats2half2_rn(w1, w1);
                    qw[kk][0] = hmul2(__byte_perm(wa, wb, 0x5410), *reinterpret_cast<const uint32_t *>(&s0));
                    qw[kk][1] = hmul2(__byte_perm(wa, wb, 0x7632), *reinterpret_cast<const uint32_t *>(&s1));
                }
            }
            const uint32_t q_addr = q_zero ? zero_addr : qb + q_row_off;
            const uint32_t q_step = q_zero ? 0u : 64u;
            const int k = x - ub;

            if (k < nri) {
                // ================= residual item: tokens t0 .. t0+n-1 in fp16
                const int t0 = k * kResTok, n = min(kResTok, r - t0);
                if (r - 1 >= t0 && r - 1 < t0 + kResTok) {   // the new token: append it to the ring
                    const int j = r - 1 - t0, part = lane >> 4, cch = lane & 15;
                    int sl = rs + r - 1;
                    if (sl >= a.ring) sl -= a.ring;
                    const uint32_t src = part == 0 ? S + kOffRk + j * 256 + 16 * (cch ^ j)
                                                   : S + kOffRv + j * 256 + 16 * ((cch + rvrot(j)) & 15);
                    const uint4 v = lds128(src);
                    *reinterpret_cast<uint4 *>((part ? a.v_res : a.k_res) + ((size_t)u * a.ring + sl) * kD + 8 * cch) =
                        v;
                }
                float sr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kq = 0; kq < 4; ++kq) {
                    uint32_t qf[4];
                    ldmatrix_x4(qf, q_addr + kq * q_step);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int kk = 2 * kq + e;
                        uint32_t ka[4];
                        ldmatrix_x4(ka, rk_live ? S + kOffRk + rk_row * 256 + 16 * ((2 * kk + (rk_m >> 1)) ^ rk_row)
                                                : zero_addr);
                        mma16816(sr, ka, qf[2 * e], qf[2 * e + 1]);
                    }
                }
                const bool valid = g_ < n;
                const float xa = valid ? sr[0] * sl2 : -INFINITY;   // absolute log2 score of token g_, head t_
                float xv = xa - m_ref;
                if (__any_sync(0xffffffffu, xv > kLazy)) {
                    const float mn = fmaxf(m_ref, warp_max_g(xa));
                    const float al = ex2(m_ref - mn);
                    l *= al;
                    pz *= al;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        acc[i][0] *= al;
                        acc[i][1] *= al;
                        acc[i][2] *= al;
                        acc[i][3] *= al;
                    }
                    m_ref = mn;
                    xv = xa - mn;
                }
                if (kMass && valid && t_ < a.g)
                    a.xs[((size_t)u * a.g + t_) * a.xs_stride + nq + t0 + g_] = xa;
                const float p = valid ? ex2(xv) : 0.f;
                l += p;
                const float ph = __half2float(__float2half_rn(p));
                const uint32_t bp = movmatrix_t(pack_half2(p, p - ph));
                // V^T fragments (m16n8k8): channel rows 16g_+I (a0) and 16g_+8+I (a1), tokens 2t_, 2t_+1
                uint4 A0 = make_uint4(0, 0, 0, 0), A1 = A0, B0 = A0, B1 = A0;
                const int ta = 2 * t_, tb = 2 * t_ + 1;
                if (ta < kResTok) {
                    const uint32_t rowa = S + kOffRv + ta * 256;
                    A0 = lds128(rowa + 16 * ((2 * g_ + rvrot(ta)) & 15));
                    A1 = lds128(rowa + 16 * ((2 * g_ + 1 + rvrot(ta)) & 15));
                }
                if (tb < kResTok) {
                    const uint32_t rowb = S + kOffRv + tb * 256;
                    B0 = lds128(rowb + 16 * ((2 * g_ + rvrot(tb)) & 15));
                    B1 = lds128(rowb + 16 * ((2 * g_ + 1 + rvrot(tb)) & 15));
                }
#define RSTEP(I)                                                                                \
    mma1688(acc[I], __byte_perm(w4(A0, I >> 1), w4(B0, I >> 1), (I & 1) ? 0x7632 : 0x5410),     \
            __byte_perm(w4(A1, I >> 1), w4(B1, I >> 1), (I & 1) ? 0x7632 : 0x5410), bp);
                RSTEP(0) RSTEP(1) RSTEP(2) RSTEP(3) RSTEP(4) RSTEP(5) RSTEP(6) RSTEP(7)
#undef RSTEP
            } else {
                // ================= packed item: tokens 32j .. 32j+31 of the unit
                const int j = k - nri;
                if (!vunit) {   // from here on acc holds packed-value units: code 2^(pos-24) per channel pair
                    vunit = true;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float f = 1.f / pair_wo(i);
                        acc[i][0] *= f;
                        acc[i][1] *= f;
                        acc[i][2] *= f;
                        acc[i][3] *= f;
                    }
                }
                // ---- zero-point term sum_c q_c z_c of head t_ (two mma, then the diagonal sum)
                float zc;
                {
                    float zd[4] = {0.f, 0.f, 0.f, 0.f};
                    uint32_t zf[4], qa0[4], qa1[4];
                    ldmatrix_x4(zf, S + zz_off);
                    ldmatrix_x4(qa0, qb + zq_off);
                    ldmatrix_x4(qa1, qb + zq_off + 128);   // chunks 4..7: c8 + 8, and (c8 + 8) ^ h = (c8 ^ h) + 8
                    mma16816(zd, qa0, zf[0], zf[1]);
                    mma16816(zd, qa1, zf[2], zf[3]);
                    float vlo = z_diag ? (z_odd ? zd[1] : zd[0]) : 0.f;   // heads 0, 1
                    float vhi = z_diag ? (z_odd ? zd[3] : zd[2]) : 0.f;   // heads 2, 3
                    vlo += __shfl_xor_sync(0xffffffffu, vlo, 4);
                    vhi += __shfl_xor_sync(0xffffffffu, vhi, 4);
                    vlo += __shfl_xor_sync(0xffffffffu, vlo, 9);
                    vhi += __shfl_xor_sync(0xffffffffu, vhi, 9);
                    const float zl = __shfl_sync(0xffffffffu, vlo, z_src), zh = __shfl_sync(0xffffffffu, vhi, z_src);
                    zc = t_ < 2 ? zl : zh;
                }
                // ---- scores: both m-tiles, one k-chunk at a time; B operand made just in time
                float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
                {
                    const uint2 ka0 = lds64(S + kOffKc + kA), kb0 = lds64(S + kOffKc + kB);
                    const uint2 ka1 = lds64(S + kOffKc + 512 + kA), kb1 = lds64(S + kOffKc + 512 + kB);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const uint32_t ksh = half ? ks_h1 : ks_h0;
                        const uint4 sA = lds128(S + kOffKs + ksh);        // channels 16w .. 16w+7, w = 2t_ + half
                        const uint4 sB = lds128(S + kOffKs + ksh + 16);   // 16w+8 .. 16w+15
                        const uint32_t a0 = half ? ka0.y : ka0.x, b0 = half ? kb0.y : kb0.x;
                        const uint32_t a1 = half ? ka1.y : ka1.x, b1 = half ? kb1.y : kb1.x;
                        const uint32_t a0r = shr10(a0), b0r = shr10(b0), a1r = shr10(a1), b1r = shr10(b1);
#define KSTEP(Q)                                                                                    \
    {                                                                                               \
        const int kk = 4 * half + Q;                                                                \
        const uint32_t e0 = __byte_perm(w4(sA, Q), w4(sB, Q), 0x5410);                              \
        const uint32_t e1 = __byte_perm(w4(sA, Q), w4(sB, Q), 0x7632);                              \
        const uint32_t bk0 = hfma2(qw[kk][0], e0, hmul2(hmul2(qw[kk][0], e0), lo_neg));             \
        const uint32_t bk1 = hfma2(qw[kk][1], e1, hmul2(hmul2(qw[kk][1], e1), lo_neg));             \
        const uint32_t f0[4] = {code_pair<2 * Q>(a0, a0r), code_pair<2 * Q>(b0, b0r),               \
                                code_pair<2 * Q + 1>(a0, a0r), code_pair<2 * Q + 1>(b0, b0r)};      \
        mma16816(s0, f0, bk0, bk1);                                                                 \
        const uint32_t f1[4] = {code_pair<2 * Q>(a1, a1r), code_pair<2 * Q>(b1, b1r),               \
                                code_pair<2 * Q + 1>(a1, a1r), code_pair<2 * Q + 1>(b1, b1r)};      \
        mma16816(s1, f1, bk0, bk1);                                                                 \
    }
                        KSTEP(0) KSTEP(1) KSTEP(2) KSTEP(3)
#undef KSTEP
                    }
                }
                // ---- x = log2 score relative to the reference max m_ref (tokens 2g_, 2g_+1, 16+2g_, 17+2g_)
                const float zcs = zc * sl2;
                const float sc[4] = {s0[0] + s0[1], s0[2] + s0[3], s1[0] + s1[1], s1[2] + s1[3]};
                float xv[4];
                {
                    const float bias = zcs - m_ref;
#pragma unroll
                    for (int i = 0; i < 4; ++i) xv[i] = fmaf(sc[i], sl2w, bias);
                }
                const float mx = fmaxf(fmaxf(xv[0], xv[1]), fmaxf(xv[2], xv[3]));
                if (__any_sync(0xffffffffu, mx > kLazy)) {
                    float xa[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) xa[i] = fmaf(sc[i], sl2w, zcs);
                    const float mn = fmaxf(m_ref, warp_max_g(fmaxf(fmaxf(xa[0], xa[1]), fmaxf(xa[2], xa[3]))));
                    const float al = ex2(m_ref - mn);
                    l *= al;
                    pz *= al;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        acc[i][0] *= al;
                        acc[i][1] *= al;
                        acc[i][2] *= al;
                        acc[i][3] *= al;
                    }
                    m_ref = mn;
#pragma unroll
                    for (int i = 0; i < 4; ++i) xv[i] = xa[i] - mn;
                }
                if (kMass && t_ < a.g) {
                    float *xrow = a.xs + ((size_t)u * a.g + t_) * a.xs_stride + (size_t)j * kSlice + 2 * g_;
                    xrow[0] = xv[0] + m_ref;
                    xrow[1] = xv[1] + m_ref;
                    xrow[16] = xv[2] + m_ref;
                    xrow[17] = xv[3] + m_ref;
                }
                // ---- P' = p * v_scale (hi / lo) and O^T += code^T P'
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    const uint32_t vsw = lds32(S + kOffVs + 2 * (16 * mt + 2 * g_));
                    const uint32_t vzw = lds32(S + kOffVz + 2 * (16 * mt + 2 * g_));
                    const float2 vsf = unpack_half2(vsw), vzf = unpack_half2(vzw);
                    const float p0 = ex2(xv[2 * mt]), p1 = ex2(xv[2 * mt + 1]);
                    l += p0 + p1;
                    pz = fmaf(p0, vzf.x, fmaf(p1, vzf.y, pz));
                    const float y0 = p0 * vsf.x, y1 = p1 * vsf.y;
                    const float2 hf = unpack_half2(pack_half2(y0, y1));
                    const uint32_t bv0 = movmatrix_t(pack_half2(y0, y0 - hf.x));
                    const uint32_t bv1 = movmatrix_t(pack_half2(y1, y1 - hf.y));
                    const uint32_t vb = S + kOffVc + 512 * mt;
                    const uint32_t wA = lds32(vb + vo0), wC = lds32(vb + vo1), wB = lds32(vb + vo2),
                                   wD = lds32(vb + vo3);
                    const uint32_t l1 = __byte_perm(wA, wB, 0x5410), h1 = __byte_perm(wA, wB, 0x7632);
                    const uint32_t l2 = __byte_perm(wC, wD, 0x5410), h2 = __byte_perm(wC, wD, 0x7632);
                    const uint32_t l1r = shr10(l1), h1r = shr10(h1), l2r = shr10(l2), h2r = shr10(h2);
#define VSTEP(NU)                                                                   \
    {                                                                               \
        const uint32_t af[4] = {code_pair<NU>(l1, l1r), code_pair<NU>(h1, h1r),     \
                                code_pair<NU>(l2, l2r), code_pair<NU>(h2, h2r)};    \
        mma16816(acc[NU], af, bv0, bv1);                                            \
    }
                    VSTEP(0) VSTEP(1) VSTEP(2) VSTEP(3) VSTEP(4) VSTEP(5) VSTEP(6) VSTEP(7)
#undef VSTEP
                }
            }
            __syncwarp();
            cstage = cstage == kStages - 1 ? 0 : cstage + 1;
            xq0 = xq1;   // the next claimed item moves to the head
            xq1 = xq2;
            --nclaim;
        }

        // ---- warp epilogue: scale to the CTA's per-head max, then
        //      y[head t_][channel] = (O^T_hi + O^T_lo) * unit + sum p * v_zero
        const float lh = warp_sum_g(l), pzh = warp_sum_g(pz);
        if (g_ == 0) sm.wm[warp][t_] = m_ref;
        __syncthreads();
        float Mc = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) Mc = fmaxf(Mc, sm.wm[w][t_]);
        const float f = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - Mc);
        const float pzf = pzh * f;
        {
            float y[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float fi = (vunit ? pair_wo(i) : 1.f) * f;
                y[i] = fmaf(acc[i][0] + acc[i][1], fi, pzf);       // channel 16g_ + i
                y[8 + i] = fmaf(acc[i][2] + acc[i][3], fi, pzf);   // channel 16g_ + 8 + i
            }
            float4 *dst = reinterpret_cast<float4 *>(&sm.wy[warp][t_][16 * g_]);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_float4(y[4 * q4], y[4 * q4 + 1], y[4 * q4 + 2], y[4 * q4 + 3]);
        }
        if (g_ == 0) sm.wl[warp][t_] = lh * f;
        finish_unit<kMass>(a, sm, sg, c - sg.first);
        if (sg.hi >= xhi) break;
        __syncthreads();   // every thread has read sm.seg and the warp states
        if (tid == 0) seg_info(a, c, sg.hi, xhi, sm.seg);
        __syncthreads();
    }
    cp_async_wait<0>();
}

// Every decode kernel lets the next kernel on the stream be placed at once:
// its CTAs take SMs as this grid's CTAs leave them and do their parameter-only
// set-up there; griddepcontrol.wait holds their first global read until this
// grid has finished and its writes are visible.
template <bool kMass>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ ArgsUni a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    launch_dependents();
    run_cta<kMass, true>(a, *reinterpret_cast<Smem *>(smem_raw), blockIdx.x);
}

// ragged batch: per-sequence lengths in the parameter table
template <bool kMass>
__global__ void __launch_bounds__(kThreads, 1) decode_ragged_kernel(const __grid_constant__ ArgsVar a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    launch_dependents();
    run_cta<kMass, true>(a, *reinterpret_cast<Smem *>(smem_raw), blockIdx.x);
}

// First flat item whose start weight is >= w, from the device-state table.
// Weights stay below 2^45, so the double divisions are exact: for integers
// N < 2^53 and D > 0, floor(fl(N / D)) = floor(N / D).
__device__ int dev_first_item(const ArgsDev &a, const long long *wbeg, long long w) {
    const int B = nseq(a);
    const int *nqa = dev_arr(a, 0), *ra = dev_arr(a, 1), *ib = dev_arr(a, 3);
    if (w >= wbeg[B]) return ib[B];
    int lo = 0, hi = B;   // largest b with wbeg[b] <= w
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (wbeg[mid] <= w) lo = mid;
        else hi = mid;
    }
    const int b = lo, nq = nqa[b], r = ra[b];
    const long long W = unit_w(nq, r);
    const long long off = w - wbeg[b];
    const int kh = (int)floor((double)off / (double)W);
    const long long rem = off - kh * W;
    return ib[b] + kh * unit_items(nq, r) + item_at(rem, unit_nri(r));
}

// Device-state mode: read the state, build the table, run the CTA's work.  The
// CTA that takes the last launch-wide ticket after reading the state writes the
// next state of every sequence (append; flush G tokens where the ring is full)
// once its items are done.  A flush that would pass `cap` is not done: the
// sequence keeps its state and its status word is set to 1.
template <bool kMass>
__global__ void __launch_bounds__(kThreads, 1) decode_dev_kernel(const ArgsDev a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    launch_dependents();
    wait_prior_grid();   // the state table is written by the previous step
    const int tid = threadIdx.x;
    const int B = nseq(a);
    int *nq = dev_arr(a, 0), *rr = dev_arr(a, 1), *rs = dev_arr(a, 2), *ib = dev_arr(a, 3), *clo = dev_arr(a, 4);
    __shared__ long long wbeg[kMaxRaggedSeqs + 1];
    int *stw = clo + a.P + 1;   // status words as read
    for (int b = tid; b < B; b += kThreads) {
        const int4 st = __ldcg(reinterpret_cast<const int4 *>(a.dseq) + b);
        nq[b] = st.x;
        rr[b] = st.y + 1;
        rs[b] = st.z;
        stw[b] = st.w;
    }
    __syncthreads();
    // The launch-wide ticket, taken as soon as the state is read (release: this
    // CTA's reads come before it) by the last thread.  Its value is first looked
    // at after the CTA's items, so the round trip is off the path to them: the
    // CTA whose ticket is the last one then writes the next state.
    unsigned ticket = 0;
    if (tid == kThreads - 1) ticket = atom_inc_acq_rel(a.grid_counter, gridDim.x - 1);
    if (tid < 32) {   // exclusive prefix sums of items and weights, 32 sequences per pass
        int ci = 0;
        long long cw = 0;
        for (int b0 = 0; b0 < B; b0 += 32) {
            const int b = b0 + tid;
            const int vi = b < B ? a.Hkv * unit_items(nq[b], rr[b]) : 0;
            const long long vw = b < B ? (long long)a.Hkv * unit_w(nq[b], rr[b]) : 0;
            int xi = vi;
            long long xw = vw;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int yi = __shfl_up_sync(0xffffffffu, xi, o);
                const long long yw = __shfl_up_sync(0xffffffffu, xw, o);
                if (tid >= o) {
                    xi += yi;
                    xw += yw;
                }
            }
            if (b < B) {
                ib[b] = ci + xi - vi;
                wbeg[b] = cw + xw - vw;
            }
            ci += __shfl_sync(0xffffffffu, xi, 31);
            cw += __shfl_sync(0xffffffffu, xw, 31);
        }
        if (tid == 0) {
            ib[B] = ci;
            wbeg[B] = cw;
            DevTab &t = dev_tab();
            t.Wt = cw;
            long long P = a.P;   // CTAs of the grid; each share at least kMinShare
            if (P > cw / kMinShare) P = cw / kMinShare;
            t.P = (int)(P < 1 ? 1 : P);
        }
    }
    __syncthreads();
    {
        const int P = dev_tab().P;
        const long long Wt = dev_tab().Wt;
        for (int cc = tid; cc <= P; cc += kThreads)
            clo[cc] = dev_first_item(a, wbeg, (long long)floor((double)cc * (double)Wt / (double)P));
    }
    __syncthreads();
    if ((int)blockIdx.x < dev_tab().P) run_cta<kMass, false>(a, *reinterpret_cast<Smem *>(smem_raw), blockIdx.x);
    // the last ticket's CTA: every sequence's new state, by its last warp (the
    // state words kept in shared memory past the CTA's own Smem)
    if (tid >= kThreads - 32 && __shfl_sync(0xffffffffu, ticket, 31) == gridDim.x - 1)
        for (int b = tid - (kThreads - 32); b < B; b += 32) {
            int4 st = make_int4(nq[b], rr[b], rs[b], stw[b]);   // a set status stays set
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

// mass[unit][t] += sum_h 2^(xs[unit][h][t] - M_h) / L_h for the n_u tokens
// the unit attended to this step (n_u, M_h, L_h from the merging CTA's stats);
// grid (ceil(max n_u / 1024), units), four consecutive tokens per thread,
// all G_ score loads issued before any use.  Launched as a programmatic
// dependent of the decode kernel: its launch overlaps the decode kernel's
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

// ------------------------------------------------------------ host planning

std::atomic<int> g_deterministic{0};   // minikv_set_deterministic

// Per-device set-up (a function attribute applies to the device current when
// it is set; the SM count is looked up per device), guarded for calls from
// several host threads.
std::mutex g_dev_mu;
bool g_attr_done[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

size_t dev_smem_bytes(int B, int P) {
    return sizeof(Smem) + sizeof(DevTab) + (5 * (size_t)B + 1 + (size_t)P + 1) * sizeof(int);
}

// the kernels' shared memory is above the 48 KB default: opt in once per device
int ensure_attr(int dev) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_attr_done[dev]) {
        const int smax = (int)dev_smem_bytes(kMaxRaggedSeqs, kMaxCtas);
        const int s = (int)sizeof(Smem);
        if (cudaFuncSetAttribute(decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, s) != cudaSuccess ||
            cudaFuncSetAttribute(decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, s) != cudaSuccess ||
            cudaFuncSetAttribute(decode_ragged_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, s) !=
                cudaSuccess ||
            cudaFuncSetAttribute(decode_ragged_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, s) !=
                cudaSuccess ||
            cudaFuncSetAttribute(decode_dev_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smax) !=
                cudaSuccess ||
            cudaFuncSetAttribute(decode_dev_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smax) !=
                cudaSuccess)
            return check_launch("decode_attn: cudaFuncSetAttribute");
        g_attr_done[dev] = true;
    }
    return MINIKV_OK;
}

// one decode CTA per SM
int sm_count(int dev) {
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        if (g_sms[dev] > 0) return g_sms[dev];
    }
    int sms = 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 148;
    cudaGetLastError();
    if (sms > kMaxCtas) sms = kMaxCtas;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    g_sms[dev] = sms;
    return sms;
}

// Host state of sequence b: the table of a ragged cache, else the shared scalars.
int seq_nq(const minikv_cache *c, int b) { return c->seq ? c->seq[3 * b] : c->n_packed; }
int seq_nres(const minikv_cache *c, int b) { return c->seq ? c->seq[3 * b + 1] : c->n_res; }
int seq_rs(const minikv_cache *c, int b) { return c->seq ? c->seq[3 * b + 2] : c->res_start; }

struct Plan {
    int units, P, S_max;
    int wu;                  // unit-boundary weight of the cut
    int max_n;               // most tokens any unit attends to this step
    std::vector<int> lo;     // host-planned modes: first item of each CTA (P + 1 entries)
};

// CTAs that take a share: one per SM, at least min_share(wu) weight each
long long cta_count(long long Wt, int slots, int wu = kWU) {
    long long P = slots;
    if (P > Wt / min_share(wu)) P = Wt / min_share(wu);
    if (P > kMaxCtas) P = kMaxCtas;
    return P < 1 ? 1 : P;
}

// Partial slots per unit for a unit of weight W when every CTA share is at
// least `share` wide: the CTA ranges its items can fall into.
int slots_bound(long long W, long long share) { return (int)(W / share + 2); }

// ---- host partition of the work list (uniform and ragged batches)
//
// The items of all units are cut into one contiguous range per CTA at equal
// steps of weight.  A unit weighs its items (kWP per packed item, kWR per
// residual item) plus a boundary weight wu placed before its first item, so a
// cut that lands in that region moves to the unit's first item and a range
// that crosses into a unit carries wu less item weight.  Which wu balances the
// CTAs best depends on the batch: with units a little larger than a share
// (Mistral-7B GQA, B=16, 6553 kept tokens; 128 units on 148 SMs) one CTA per
// unit and no split is fastest, with many small units or a ragged batch a
// small wu is.  So each call takes, from a few candidates, the wu whose cuts
// minimise a cost model of the slowest CTA: the weight of its items, plus
// kSegCost for every unit it works on (the end of a segment), plus kSplitCost
// for every unit it shares with another CTA (partial write, arrival, merge).
// The two costs were fitted to measured launch times of five batch shapes at
// boundary weights from 0 to 2^20; with them the model ranks each shape's
// fastest measured weight first.
constexpr int kWuCand[] = {128, 256, 512, 896, 1280, 1 << 20};
constexpr long long kSegCost = 120, kSplitCost = 200;

struct Shape {              // per-sequence state of this call (n_q, r = residual tokens + the new one)
    int B, Hkv;
    std::vector<int> nq, r, ibeg;
};

// Cuts of the work list for boundary weight wu: P, S_max and lo of p.
void cut(const Shape &s, int wu, int sms, Plan &p) {
    std::vector<long long> wbeg(s.B + 1, 0);
    long long Wmax = 0;
    for (int b = 0; b < s.B; ++b) {
        const long long W = unit_w(s.nq[b], s.r[b], wu);
        if (W > Wmax) Wmax = W;
        wbeg[b + 1] = wbeg[b] + (long long)s.Hkv * W;
    }
    const long long Wt = wbeg[s.B];
    p.P = (int)cta_count(Wt, sms, wu);
    p.S_max = slots_bound(Wmax, Wt / p.P);
    if (p.S_max > p.P) p.S_max = p.P;
    // first item whose start weight is >= floor(i Wt / P), for each CTA boundary i
    p.lo.resize(p.P + 1);
    int b = 0;
    for (int i = 0; i <= p.P; ++i) {
        const long long w = (long long)((__int128)i * Wt / p.P);
        if (w >= Wt) {
            p.lo[i] = s.ibeg[s.B];
            continue;
        }
        while (wbeg[b + 1] <= w) ++b;
        const long long W = unit_w(s.nq[b], s.r[b], wu);
        const long long off = w - wbeg[b];
        const int kh = (int)(off / W);
        const long long rem = off - kh * W;
        p.lo[i] = s.ibeg[b] + kh * unit_items(s.nq[b], s.r[b]) + item_at(rem, unit_nri(s.r[b]), wu);
    }
}

// Modelled cost of the slowest CTA of a cut (see above); stops early once it
// reaches `stop` (a cost that cannot win), if stop >= 0.
long long slowest_cta(const Shape &s, const Plan &p, long long stop) {
    long long worst = 0;
    int b = 0, kh = 0;   // the unit that holds lo[c]
    for (int c = 0; c < p.P; ++c) {
        const int x0 = p.lo[c], x1 = p.lo[c + 1];
        if (x0 >= x1) continue;
        for (;;) {
            const int n = unit_items(s.nq[b], s.r[b]);
            if (x0 < s.ibeg[b] + (kh + 1) * n) break;
            if (++kh == s.Hkv) {
                kh = 0;
                ++b;
            }
        }
        long long cost = 0;
        for (int bb = b, kk = kh; bb < s.B;) {
            const int n = unit_items(s.nq[bb], s.r[bb]), nri = unit_nri(s.r[bb]);
            const int us = s.ibeg[bb] + kk * n, ue = us + n;
            if (us >= x1) break;
            const int lo = x0 > us ? x0 : us, hi = x1 < ue ? x1 : ue;
            int res = (hi < us + nri ? hi : us + nri) - lo;
            if (res < 0) res = 0;
            cost += (long long)res * kWR + (long long)(hi - lo - res) * kWP + kSegCost;
            if (lo > us || hi < ue) cost += kSplitCost;
            if (++kk == s.Hkv) {
                kk = 0;
                ++bb;
            }
        }
        if (cost > worst) worst = cost;
        if (stop >= 0 && worst >= stop) return worst;
    }
    return worst;
}

// The boundary weight of the cheapest modelled cut; ties go to the smaller
// weight.  The model is evaluated with each sequence's residual count r moved
// to the middle of its 32-token bucket (it moves the choice little, and a
// batch then keeps its weight for up to 32 steps).  A pure function of the
// call's state, so the same state always gets the same cut; a small cache per
// host thread, keyed by the bucketed state, saves the search.
int choose_wu(const Shape &s, int sms, bool uniform, int ring) {
    std::vector<int> key;
    key.reserve(5 + 2 * s.B);
    key.push_back(sms);
    key.push_back(s.Hkv);
    key.push_back(s.B);
    key.push_back(uniform ? 1 : 0);
    for (int b = 0; b < (uniform ? 1 : s.B); ++b) {
        key.push_back(s.nq[b]);
        key.push_back(s.r[b] >> 5);
    }
    thread_local std::map<std::vector<int>, int> memo;
    const auto it = memo.find(key);
    if (it != memo.end()) return it->second;
    Shape m = s;   // the bucketed state
    for (int b = 0; b < s.B; ++b) {
        const int rc = (s.r[b] >> 5) * 32 + 16;
        m.r[b] = rc < 1 ? 1 : rc > ring ? ring : rc;
        m.ibeg[b + 1] = m.ibeg[b] + s.Hkv * unit_items(m.nq[b], m.r[b]);
    }
    int best_wu = kWU;
    long long best = -1;
    Plan p;
    for (const int wu : kWuCand) {
        cut(m, wu, sms, p);
        const long long v = slowest_cta(m, p, best);
        if (best < 0 || v < best) {
            best = v;
            best_wu = wu;
        }
    }
    if (memo.size() >= 256) memo.clear();
    memo.emplace(std::move(key), best_wu);
    return best_wu;
}

Plan plan(const minikv_cache *c, int dev) {
    Plan p;
    p.units = c->B * c->Hkv;
    const int ring = c->R + c->G;
    if (c->dseq) {
        // device-state mode: one configuration for every state the cache can hold;
        // the kernel partitions this step's items itself, at boundary weight kWU
        const long long Wmax = unit_w(c->cap, ring);
        p.P = (int)cta_count((long long)p.units * Wmax, sm_count(dev));
        p.S_max = slots_bound(Wmax, kMinShare);
        if (p.S_max > p.P) p.S_max = p.P;
        p.max_n = c->cap + ring;
        p.wu = kWU;
        return p;
    }
    const bool ragged = c->seq != nullptr;
    Shape s;
    s.B = c->B;
    s.Hkv = c->Hkv;
    s.nq.resize(c->B);
    s.r.resize(c->B);
    s.ibeg.assign(c->B + 1, 0);
    p.max_n = 0;
    for (int b = 0; b < c->B; ++b) {
        const int q = ragged ? b : 0;
        s.nq[b] = seq_nq(c, q);
        s.r[b] = seq_nres(c, q) + 1;
        if (s.nq[b] + s.r[b] > p.max_n) p.max_n = s.nq[b] + s.r[b];
        s.ibeg[b + 1] = s.ibeg[b] + c->Hkv * unit_items(s.nq[b], s.r[b]);
    }
    const int sms = sm_count(dev);
    p.wu = choose_wu(s, sms, !ragged, ring);
    cut(s, p.wu, sms, p);
    return p;
}

}  // namespace

// Bytes of the workspace prefix that holds the per-unit arrival counters and
// the launch-wide counter of the device-state mode.
size_t decode_counter_bytes(int B, int Hkv) { return (((size_t)B * Hkv * 4 + 4 + 255) / 256) * 256; }

// Partial slots per unit for any state up to max_tokens tokens per unit: each
// CTA share is at least kMinShare weight, so a unit of weight W meets at most
// W / kMinShare + 2 CTAs.
static size_t slots_for(int max_tokens) {
    const int res_max = max_tokens < 1024 ? max_tokens : 1024;   // the ring holds at most 1024 tokens
    const long long W = unit_w(max_tokens, res_max < 1 ? 1 : res_max);
    long long s = W / kMinShare + 2;
    if (s > kMaxCtas) s = kMaxCtas;
    return (size_t)s;
}

size_t decode_workspace_bytes(int B, int Hkv, int max_tokens) {
    const size_t units = (size_t)B * Hkv;
    return decode_counter_bytes(B, Hkv) + units * slots_for(max_tokens) * 4 * kPartStride * 4;
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

void decode_set_deterministic(int on) { g_deterministic.store(on ? 1 : 0, std::memory_order_relaxed); }

// The launch the next decode call on this cache state makes: CTAs, boundary
// weight and (host-planned modes, n_first >= P + 1) each CTA's first item.
int decode_plan_info(const minikv_cache *c, int *ctas, int *wu, int *first, int n_first) {
    const int dev = current_device();
    const Plan p = plan(c, dev < 0 ? 0 : dev);
    *ctas = p.P;
    *wu = p.wu;
    if (first && !c->dseq) {
        if (n_first < p.P + 1)
            return fail(MINIKV_ERR_INVALID_ARG, "decode_plan: first_items needs %d entries, %d given", p.P + 1,
                        n_first);
        for (int i = 0; i <= p.P; ++i) first[i] = p.lo[i];
    }
    return MINIKV_OK;
}

// Workspace bytes the next decode call on this cache state will use.
size_t decode_call_workspace_bytes(const minikv_cache *c) {
    const int dev = current_device();
    const Plan p = plan(c, dev < 0 ? 0 : dev);
    return decode_counter_bytes(c->B, c->Hkv) + (size_t)p.units * p.S_max * 4 * kPartStride * 4;
}

namespace {

// Every decode launch is a programmatic dependent of the work before it on the
// stream: its CTAs may be placed while the previous kernel drains, and
// griddepcontrol.wait at their top holds them until that kernel has finished
// and its writes are visible.
template <class K, class A>
int launch_pdl(K kernel, const A &a, int grid, size_t smem, cudaStream_t stream, const char *what) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, a);
    return check_launch(what);
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
    const int dev = current_device();
    if (dev < 0) return fail(MINIKV_ERR_CUDA, "decode_attn: no current CUDA device");
    const int arc = ensure_attr(dev);
    if (arc) return arc;
    const Plan p = plan(c, dev);
    const size_t cnt_bytes = decode_counter_bytes(c->B, c->Hkv);
    const size_t part_bytes = (size_t)p.units * p.S_max * 4 * kPartStride * 4;
    size_t need = cnt_bytes + part_bytes;
    if (mass) need += mass_stats_bytes(c->B, c->Hkv) + mass_scores_bytes(c->B, c->Hkv, g, p.max_n);
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
    a.grid_counter = a.counters + p.units;
    a.dseq = c->dseq;
    a.part = reinterpret_cast<float *>(static_cast<char *>(ws) + cnt_bytes);
    a.stats = mass ? reinterpret_cast<float *>(static_cast<char *>(ws) + cnt_bytes + part_bytes) : nullptr;
    a.xs = mass ? reinterpret_cast<float *>(static_cast<char *>(ws) + cnt_bytes + part_bytes +
                                            mass_stats_bytes(c->B, c->Hkv))
                : nullptr;
    a.xs_stride = (p.max_n + 3) & ~3;
    a.Hkv = c->Hkv; a.g = g; a.G = c->G; a.cap = c->cap; a.ring = ring;
    a.n_q = c->n_packed; a.r = c->n_res + 1; a.res_start = c->res_start;
    a.groups_cap = c->cap / c->G;
    a.lg2G = 31 - __builtin_clz((unsigned)c->G);
    a.units = p.units; a.P = p.P; a.S_max = p.S_max;
    a.nb = c->B;
    a.scale_log2 = sm_scale * kLog2e;
    a.det = g_deterministic.load(std::memory_order_relaxed);

    int rc;
    if (c->dseq) {
        ArgsDev ad;
        static_cast<Args &>(ad) = a;
        const size_t smem = dev_smem_bytes(c->B, p.P);
        rc = mass ? launch_pdl(decode_dev_kernel<true>, ad, p.P, smem, stream, "decode_attn_mass (device state)")
                  : launch_pdl(decode_dev_kernel<false>, ad, p.P, smem, stream, "decode_attn (device state)");
        if (rc) return rc;
        return mass ? launch_mass(a, p, mass, (long long)c->cap + ring, stream) : MINIKV_OK;
    } else if (c->seq) {
        ArgsVar av;
        static_cast<Args &>(av) = a;
        av.tab.ibeg[0] = 0;
        for (int b = 0; b < c->B; ++b) {
            const int nq = seq_nq(c, b), r = seq_nres(c, b) + 1;
            av.tab.n_q[b] = nq;
            av.tab.r[b] = r;
            av.tab.res_start[b] = seq_rs(c, b);
            av.tab.ibeg[b + 1] = av.tab.ibeg[b] + c->Hkv * unit_items(nq, r);
        }
        for (int i = 0; i <= p.P; ++i) av.cta.lo[i] = p.lo[i];
        rc = mass ? launch_pdl(decode_ragged_kernel<true>, av, p.P, sizeof(Smem), stream, "decode_attn_mass (ragged)")
                  : launch_pdl(decode_ragged_kernel<false>, av, p.P, sizeof(Smem), stream, "decode_attn (ragged)");
    } else {
        ArgsUni au;
        static_cast<Args &>(au) = a;
        for (int i = 0; i <= p.P; ++i) au.cta.lo[i] = p.lo[i];
        rc = mass ? launch_pdl(decode_kernel<true>, au, p.P, sizeof(Smem), stream, "decode_attn_mass")
                  : launch_pdl(decode_kernel<false>, au, p.P, sizeof(Smem), stream, "decode_attn");
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
