// minikv_topk_evict: keep the observation window plus the highest-scoring
// earlier tokens, then gather their K/V rows.
//
// Source: gptget.net summary of arXiv 2411.18077, glossary 术语表 "adaptive
// KV" (keep the KV states that matter, by importance) and the LongBench table
// of pre.notesum.ai ("MiniKV Pyramid": a different budget per layer, chosen by
// the caller through `keep`).
//
// select_kernel: one CTA (1024 threads) per (b, KV head) row.  An exact radix
// select (4 passes of 8 bits over order-preserving keys of the fp32 scores)
// finds the (keep-W)-th largest candidate score u*; positions with score > u*
// are kept, plus the lowest-index positions with score == u* (ties go to the
// lower index), plus the window.  An ordered block scan writes them ascending.
// gather_kernel: 16-byte row copies of the kept K and V rows.
#include "common.cuh"

namespace minikv {

namespace {

constexpr int kSelThreads = 1024;

// Order-preserving unsigned key of an fp32 score.  -0 and +0 are one value
// (the selection compares scores as numbers), so -0 is first made +0.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(__fadd_rn(f, 0.0f));
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix of `flag` over the block in thread order; returns the
// prefix and writes the block total to *total.  Uses `warp_tot` [32] smem.
__device__ __forceinline__ int block_scan(bool flag, int *warp_tot, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned bal = __ballot_sync(0xffffffffu, flag);
    const int in_warp = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) warp_tot[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
        int v = warp_tot[lane];
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        warp_tot[lane] = x - v;   // exclusive
        if (lane == 31) warp_tot[32] = x;
    }
    __syncthreads();
    const int res = warp_tot[warp] + in_warp;
    *total = warp_tot[32];
    __syncthreads();
    return res;
}

struct SelArgs {
    const float *scores;
    int32_t *idx;
    int T, W, keep;
};

__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelArgs a) {
    __shared__ int hist[256];
    __shared__ int warp_tot[33];
    __shared__ uint32_t s_prefix;
    __shared__ int s_need;
    const int tid = threadIdx.x;
    const int row = blockIdx.x;
    const float *s = a.scores + (size_t)row * a.T;
    const int n_out = a.keep < a.T ? a.keep : a.T;
    int32_t *out = a.idx + (size_t)row * n_out;

    if (a.keep >= a.T) {
        for (int j = tid; j < a.T; j += kSelThreads) out[j] = j;
        return;
    }
    const int nc = a.T - a.W;       // candidates [0, nc)
    const int k1 = a.keep - a.W;    // how many of them to keep
    uint32_t prefix = 0, pmask = 0;
    int need = k1;                  // still to take at the current prefix
    if (k1 > 0) {
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
            __syncthreads();
            for (int j = tid; j < nc; j += kSelThreads) {
                const uint32_t u = order_key(s[j]);
                if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255], 1);
            }
            __syncthreads();
            if (tid < 32) {
                // lane l owns bins 255-8l .. 248-8l (descending); suffix counts from the top
                int loc = 0;
                for (int i = 0; i < 8; ++i) loc += hist[255 - 8 * tid - i];
                int incl = loc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (tid >= o) incl += y;
                }
                const int excl = incl - loc;
                const bool mine = excl < need && incl >= need;
                if (mine) {
                    int cum = excl;
                    for (int i = 0; i < 8; ++i) {
                        const int bin = 255 - 8 * tid - i;
                        if (cum + hist[bin] >= need) {
                            s_prefix = prefix | ((uint32_t)bin << shift);
                            s_need = need - cum;
                            break;
                        }
                        cum += hist[bin];
                    }
                }
            }
            __syncthreads();
            prefix = s_prefix;
            need = s_need;
            pmask |= 255u << shift;
            __syncthreads();
        }
    }
    // ordered compaction: keep j if j in window, or key > u*, or key == u* and
    // it is among the first `need` equal keys by index
    int base = 0, eq_base = 0;
    for (int j0 = 0; j0 < a.T; j0 += kSelThreads) {
        const int j = j0 + tid;
        bool in = j < a.T;
        bool eq = false, keepit = false;
        if (in) {
            if (j >= nc) keepit = true;
            else if (k1 > 0) {
                const uint32_t u = order_key(s[j]);
                keepit = u > prefix;
                eq = (u == prefix);
            }
        }
        int eq_tot;
        const int eq_rank = eq_base + block_scan(eq, warp_tot, &eq_tot);
        eq_base += eq_tot;
        if (eq && eq_rank < need) keepit = true;
        int tot;
        const int pos = base + block_scan(keepit, warp_tot, &tot);
        if (keepit && pos < n_out) out[pos] = j;
        base += tot;
    }
}

struct GatherArgs {
    const int32_t *idx;
    const uint16_t *k, *v;
    uint16_t *kk, *vk;
    int T, n;
};

__global__ void __launch_bounds__(128) gather_kernel(const GatherArgs a) {
    const int unit = blockIdx.y;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 4);
    const int ch = threadIdx.x & 15;
    if (r >= a.n) return;
    const int j = a.idx[(size_t)unit * a.n + r];
    if ((unsigned)j >= (unsigned)a.T) return;
    const size_t src = ((size_t)unit * a.T + j) * kD;
    const size_t dst = ((size_t)unit * a.n + r) * kD;
    reinterpret_cast<uint4 *>(a.kk + dst)[ch] = reinterpret_cast<const uint4 *>(a.k + src)[ch];
    reinterpret_cast<uint4 *>(a.vk + dst)[ch] = reinterpret_cast<const uint4 *>(a.v + src)[ch];
}

}  // namespace

int select_launch(const float *scores, int B, int Hkv, int T, int W, int keep, int32_t *idx, cudaStream_t stream) {
    SelArgs sa{scores, idx, T, W, keep};
    select_kernel<<<B * Hkv, kSelThreads, 0, stream>>>(sa);
    return check_launch("topk_evict: select");
}

int topk_launch(const float *scores, const uint16_t *k, const uint16_t *v, int B, int Hkv, int T, int W, int keep,
                int32_t *idx, uint16_t *k_kept, uint16_t *v_kept, cudaStream_t stream) {
    const int units = B * Hkv;
    int rc = select_launch(scores, B, Hkv, T, W, keep, idx, stream);
    if (rc) return rc;
    const int n = keep < T ? keep : T;
    GatherArgs ga{idx, k, v, k_kept, v_kept, T, n};
    gather_kernel<<<dim3((n + 7) / 8, units), 128, 0, stream>>>(ga);
    return check_launch("topk_evict: gather");
}

}  // namespace minikv
