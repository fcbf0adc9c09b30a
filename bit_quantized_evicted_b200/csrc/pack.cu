// minikv_quant_pack: quantize a compacted kept sequence into the 2-bit cache.
//
// Source: gptget.net summary of arXiv 2411.18077, section 方法论 / 方法详解:
// sub-channel (per-channel) key quantization and per-token value quantization
// into a compact layout.  The newest r tokens stay fp16 in the residual ring.
//
// Grid (n_groups + n_res_blocks, B*Hkv), 128 threads.  Block x < n_groups packs
// key group x and the same G value tokens: it first stages the G key and value
// rows in shared memory (cp.async, all in flight), then quantizes from there;
// the remaining blocks copy residual tokens into ring slots 0..r-1.
// Memory-bound: 512 B read and 84 B written per packed token and KV head.
//
// minikv_evict_pack runs the same kernel with an index list: compacted token
// t of a unit is then prompt row idx[t] (the kept positions of
// minikv_topk_evict), read straight from the prompt K/V, so the kept rows are
// never written out in fp16 (the fused select -> gather -> pack of the path).
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
};

constexpr int kResPerBlock = 32;   // residual tokens copied per block
constexpr int kStageG = 64;        // key groups up to this size are staged in shared memory (32 KB)

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
        if (a.G <= kStageG) {
            // stage the group's G key rows and G value rows in shared memory
            // (swizzled), every 16-byte copy in flight at once, then pack from there
            extern __shared__ __align__(16) uint16_t tile[];   // [2][G][128]
            uint16_t *kt = tile, *vt = tile + a.G * kD;
            for (int e = threadIdx.x; e < a.G * 16; e += 128) {
                const int t = e >> 4, ch = e & 15;
                const size_t src = src_row(t0 + t) * kD + ch * 8;
                cp_async16(smem_addr(kt + swz(t, ch * 8)), ku + src, true);
                cp_async16(smem_addr(vt + swz(t, ch * 8)), vu + src, true);
            }
            cp_async_commit();
            cp_async_wait<0>();
            __syncthreads();
            auto kat = [&](int t, int c) -> const uint16_t * { return kt + swz(t, c); };
            auto vat = [&](int t, int c) -> const uint16_t * { return vt + swz(t, c); };
            pack_key_group(kat, a.G, a.k_codes + tok * 8, a.k_scale + grow * kD, a.k_zero + grow * kD, scr);
            pack_value_tokens(vat, a.G, a.Gv, a.v_codes + tok * 8, a.v_scale + tok * (kD / a.Gv),
                              a.v_zero + tok * (kD / a.Gv));
        } else {
            auto krow = [&](int t, int c) { return ku + src_row(t0 + t) * kD + c; };
            auto vrow = [&](int t, int c) { return vu + src_row(t0 + t) * kD + c; };
            pack_key_group(krow, a.G, a.k_codes + tok * 8, a.k_scale + grow * kD, a.k_zero + grow * kD, scr);
            pack_value_tokens(vrow, a.G, a.Gv, a.v_codes + tok * 8, a.v_scale + tok * (kD / a.Gv),
                              a.v_zero + tok * (kD / a.Gv));
        }
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
    int gx = a.n_groups + n_res_blocks;
    if (c->dseq && gx == 0) gx = 1;   // an empty load still sets the device state
    const int units = seq >= 0 ? c->Hkv : c->B * c->Hkv;
    if (gx > 0 && units > 0) {
        const size_t smem = c->G <= kStageG ? (size_t)2 * c->G * kD * sizeof(uint16_t) : 0;
        pack_kernel<<<dim3(gx, units), 128, smem, stream>>>(a);
        int rc = check_launch("quant_pack");
        if (rc) return rc;
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
