// C ABI of libminikv: argument validation, error strings, cache carving, and
// dispatch to the kernels of pack.cu, prefill.cu, topk.cu and decode.cu.
#include <stdarg.h>
#include <stdio.h>

#include "common.cuh"

namespace minikv {

static thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return code;
}

int check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(MINIKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return MINIKV_OK;
}

int pack_launch(minikv_cache *c, const uint16_t *k, const uint16_t *v, int N, cudaStream_t stream,
                const int32_t *idx = nullptr, int T = 0, int seq = -1);
int select_launch(const float *scores, int B, int Hkv, int T, int W, int keep, int32_t *idx, cudaStream_t stream);
int prefill_launch(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int Hq, int Hkv, int T, int W,
                   float sm_scale, uint16_t *o, float *scores, void *ws, cudaStream_t stream);
size_t prefill_workspace_bytes(int B, int Hq, int W);
size_t prefill_lse_bytes(int B, int Hq, int W);
int topk_launch(const float *scores, const uint16_t *k, const uint16_t *v, int B, int Hkv, int T, int W, int keep,
                int32_t *idx, uint16_t *k_kept, uint16_t *v_kept, cudaStream_t stream);
int decode_launch(minikv_cache *c, const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new, int Hq,
                  float sm_scale, uint16_t *out, void *ws, size_t ws_bytes, cudaStream_t stream,
                  float *mass = nullptr);
size_t decode_workspace_bytes(int B, int Hkv, int max_tokens);
size_t decode_mass_workspace_bytes(int B, int Hq, int Hkv, int max_tokens);
void decode_set_deterministic(int on);
int decode_plan_info(const minikv_cache *c, int *ctas, int *wu, int *first, int n_first);

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// shape rules shared by the cache-level calls
static int check_cache_shape(int B, int Hkv, int D, int G, int Gv, int R, int cap) {
    if (B < 1 || Hkv < 1 || G < 1 || Gv < 1 || R < 0 || cap < 0)
        return fail(MINIKV_ERR_INVALID_ARG, "cache shape: B=%d Hkv=%d G=%d Gv=%d R=%d cap=%d", B, Hkv, G, Gv, R, cap);
    if (D != kD) return fail(MINIKV_ERR_UNSUPPORTED, "head size D=%d (only 128)", D);
    if (!(G == 32 || G == 64 || G == 128)) return fail(MINIKV_ERR_UNSUPPORTED, "key group G=%d (32, 64 or 128)", G);
    if (!(Gv == 16 || Gv == 32 || Gv == 64 || Gv == 128))
        return fail(MINIKV_ERR_UNSUPPORTED, "value group Gv=%d (16, 32, 64 or 128)", Gv);
    if (cap % G != 0) return fail(MINIKV_ERR_INVALID_ARG, "cap=%d is not a multiple of G=%d", cap, G);
    if (R + G > 1024) return fail(MINIKV_ERR_UNSUPPORTED, "residual ring R+G=%d above 1024", R + G);
    return MINIKV_OK;
}

static int check_cache(const minikv_cache *c) {
    if (!c) return fail(MINIKV_ERR_INVALID_ARG, "null cache");
    int rc = check_cache_shape(c->B, c->Hkv, c->D, c->G, c->Gv, c->R, c->cap);
    if (rc) return rc;
    const void *ptrs[8] = {c->k_codes, c->v_codes, c->k_scale, c->k_zero, c->v_scale, c->v_zero, c->k_res, c->v_res};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return fail(MINIKV_ERR_INVALID_ARG, "cache array null or not 16-byte aligned");
    auto bad_state = [&](int n_packed, int n_res, int res_start) {
        return n_packed < 0 || n_packed % c->G || n_packed > c->cap || n_res < 0 || n_res >= c->R + c->G ||
               res_start < 0 || res_start >= c->R + c->G;
    };
    if (c->dseq) {
        if (c->B > MINIKV_MAX_RAGGED_SEQS)
            return fail(MINIKV_ERR_UNSUPPORTED, "device-state cache with B=%d above %d", c->B, MINIKV_MAX_RAGGED_SEQS);
    } else if (c->seq) {
        if (c->B > MINIKV_MAX_RAGGED_SEQS)
            return fail(MINIKV_ERR_UNSUPPORTED, "ragged cache with B=%d above %d", c->B, MINIKV_MAX_RAGGED_SEQS);
        for (int b = 0; b < c->B; ++b)
            if (bad_state(c->seq[3 * b], c->seq[3 * b + 1], c->seq[3 * b + 2]))
                return fail(MINIKV_ERR_INVALID_ARG, "state of sequence %d: n_packed=%d n_res=%d res_start=%d", b,
                            c->seq[3 * b], c->seq[3 * b + 1], c->seq[3 * b + 2]);
    } else if (bad_state(c->n_packed, c->n_res, c->res_start)) {
        return fail(MINIKV_ERR_INVALID_ARG, "cache state n_packed=%d n_res=%d res_start=%d", c->n_packed, c->n_res,
                    c->res_start);
    }
    return MINIKV_OK;
}

// The argument checks of minikv_decode_attn other than the workspace, for
// entry points that bring their own scratch.
int decode_validate(minikv_cache *c, const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new, int Hq,
                    const uint16_t *out) {
    g_err[0] = 0;
    int rc = check_cache(c);
    if (rc) return rc;
    if (!q || !k_new || !v_new || !out) return fail(MINIKV_ERR_INVALID_ARG, "decode_attn: null pointer");
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out))
        return fail(MINIKV_ERR_INVALID_ARG, "decode_attn: pointers must be 16-byte aligned");
    if (Hq < 1 || Hq % c->Hkv) return fail(MINIKV_ERR_INVALID_ARG, "decode_attn: Hq=%d, Hkv=%d", Hq, c->Hkv);
    if (Hq / c->Hkv > 4) return fail(MINIKV_ERR_UNSUPPORTED, "decode_attn: more than 4 query heads per KV head");
    if (c->Gv != c->D) return fail(MINIKV_ERR_UNSUPPORTED, "decode_attn: value group Gv=%d (needs Gv = D)", c->Gv);
    if ((size_t)c->B * c->Hkv > 65535) return fail(MINIKV_ERR_UNSUPPORTED, "decode_attn: B*Hkv above 65535");
    if ((size_t)c->B * c->Hkv * (c->cap / 32 + (c->R + c->G + 4) / 5) >= (1u << 31))
        return fail(MINIKV_ERR_UNSUPPORTED, "decode_attn: B*Hkv*(cap/32 + (R+G)/5) must stay below 2^31");
    const int nb = c->dseq ? 0 : (c->seq ? c->B : 1);   // a device-resident state is checked on the device
    for (int b = 0; b < nb; ++b) {
        const int n_packed = c->seq ? c->seq[3 * b] : c->n_packed, n_res = c->seq ? c->seq[3 * b + 1] : c->n_res;
        if (n_res + 1 == c->R + c->G && n_packed + c->G > c->cap)
            return fail(MINIKV_ERR_CAPACITY, "decode_attn: flushing a key group of sequence %d would exceed cap=%d",
                        b, c->cap);
    }
    return MINIKV_OK;
}

}  // namespace minikv

using namespace minikv;

extern "C" {

const char *minikv_last_error_string(void) { return g_err; }

size_t minikv_cache_bytes(int B, int Hkv, int D, int G, int Gv, int R, int cap) {
    if (check_cache_shape(B, Hkv, D, G, Gv, R, cap)) return 0;
    const size_t u = (size_t)B * Hkv;
    const size_t codes = up256(u * cap * (D / 16) * 4);
    const size_t kscale = up256(u * (cap / G) * D * 2);
    const size_t vscale = up256(u * cap * (D / Gv) * 2);
    const size_t res = up256(u * (R + G) * D * 2);
    return 2 * codes + 2 * kscale + 2 * vscale + 2 * res;
}

int minikv_cache_bind(minikv_cache *c, void *base, size_t bytes, int B, int Hkv, int D, int G, int Gv, int R,
                      int cap) {
    g_err[0] = 0;
    if (!c || !base) return fail(MINIKV_ERR_INVALID_ARG, "cache_bind: null pointer");
    int rc = check_cache_shape(B, Hkv, D, G, Gv, R, cap);
    if (rc) return rc;
    if (reinterpret_cast<uintptr_t>(base) & 255u)
        return fail(MINIKV_ERR_INVALID_ARG, "cache_bind: base not 256-byte aligned");
    const size_t need = minikv_cache_bytes(B, Hkv, D, G, Gv, R, cap);
    if (bytes < need) return fail(MINIKV_ERR_INVALID_ARG, "cache_bind: %zu bytes needed, %zu given", need, bytes);
    const size_t u = (size_t)B * Hkv;
    char *p = static_cast<char *>(base);
    auto take = [&](size_t n) { char *r = p; p += up256(n); return r; };
    c->B = B; c->Hkv = Hkv; c->D = D; c->G = G; c->Gv = Gv; c->R = R; c->cap = cap;
    c->k_codes = reinterpret_cast<uint32_t *>(take(u * cap * (D / 16) * 4));
    c->v_codes = reinterpret_cast<uint32_t *>(take(u * cap * (D / 16) * 4));
    c->k_scale = reinterpret_cast<uint16_t *>(take(u * (cap / G) * D * 2));
    c->k_zero = reinterpret_cast<uint16_t *>(take(u * (cap / G) * D * 2));
    c->v_scale = reinterpret_cast<uint16_t *>(take(u * cap * (D / Gv) * 2));
    c->v_zero = reinterpret_cast<uint16_t *>(take(u * cap * (D / Gv) * 2));
    c->k_res = reinterpret_cast<uint16_t *>(take(u * (R + G) * D * 2));
    c->v_res = reinterpret_cast<uint16_t *>(take(u * (R + G) * D * 2));
    c->n_packed = 0; c->n_res = 0; c->res_start = 0;
    c->seq = nullptr;
    c->dseq = nullptr;
    return MINIKV_OK;
}

int minikv_cache_set_device_state(minikv_cache *c, int *dseq, void *stream) {
    g_err[0] = 0;
    if (!c) return fail(MINIKV_ERR_INVALID_ARG, "cache_set_device_state: null cache");
    if (dseq) {
        if (c->B < 1 || c->B > MINIKV_MAX_RAGGED_SEQS)
            return fail(MINIKV_ERR_UNSUPPORTED, "cache_set_device_state: B=%d (1..%d)", c->B, MINIKV_MAX_RAGGED_SEQS);
        if (!aligned16(dseq)) return fail(MINIKV_ERR_INVALID_ARG, "cache_set_device_state: dseq not 16-byte aligned");
        cudaError_t e = cudaMemsetAsync(dseq, 0, (size_t)c->B * 4 * sizeof(int), static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess)
            return fail(MINIKV_ERR_CUDA, "cache_set_device_state: clearing the state: %s", cudaGetErrorString(e));
    }
    c->dseq = dseq;
    c->n_packed = 0; c->n_res = 0; c->res_start = 0;
    if (c->seq)
        for (int i = 0; i < 3 * c->B; ++i) c->seq[i] = 0;
    return MINIKV_OK;
}

int minikv_cache_set_ragged(minikv_cache *c, int *seq) {
    g_err[0] = 0;
    if (!c) return fail(MINIKV_ERR_INVALID_ARG, "cache_set_ragged: null cache");
    if (seq && (c->B < 1 || c->B > MINIKV_MAX_RAGGED_SEQS))
        return fail(MINIKV_ERR_UNSUPPORTED, "cache_set_ragged: B=%d (1..%d)", c->B, MINIKV_MAX_RAGGED_SEQS);
    c->seq = seq;
    c->n_packed = 0; c->n_res = 0; c->res_start = 0;
    if (seq)
        for (int i = 0; i < 3 * c->B; ++i) seq[i] = 0;
    return MINIKV_OK;
}

int minikv_quant_pack(minikv_cache *c, const uint16_t *k, const uint16_t *v, int n_tokens, void *stream) {
    g_err[0] = 0;
    int rc = check_cache(c);
    if (rc) return rc;
    if (n_tokens < 0) return fail(MINIKV_ERR_INVALID_ARG, "quant_pack: n_tokens=%d", n_tokens);
    if (n_tokens > 0 && (!k || !v || !aligned16(k) || !aligned16(v)))
        return fail(MINIKV_ERR_INVALID_ARG, "quant_pack: k/v null or not 16-byte aligned");
    return pack_launch(c, k, v, n_tokens, static_cast<cudaStream_t>(stream));
}

int minikv_quant_pack_seq(minikv_cache *c, int b, const uint16_t *k, const uint16_t *v, int n_tokens,
                          void *stream) {
    g_err[0] = 0;
    int rc = check_cache(c);
    if (rc) return rc;
    if (!c->seq && !c->dseq) return fail(MINIKV_ERR_INVALID_ARG, "quant_pack_seq: the cache is not ragged");
    if (b < 0 || b >= c->B) return fail(MINIKV_ERR_INVALID_ARG, "quant_pack_seq: sequence %d of %d", b, c->B);
    if (n_tokens < 0) return fail(MINIKV_ERR_INVALID_ARG, "quant_pack_seq: n_tokens=%d", n_tokens);
    if (n_tokens > 0 && (!k || !v || !aligned16(k) || !aligned16(v)))
        return fail(MINIKV_ERR_INVALID_ARG, "quant_pack_seq: k/v null or not 16-byte aligned");
    return pack_launch(c, k, v, n_tokens, static_cast<cudaStream_t>(stream), nullptr, 0, b);
}

int minikv_select_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int Hq, int Hkv, int T,
                          int D, int W, float sm_scale, uint16_t *o, float *scores, void *ws, size_t ws_bytes,
                          void *stream) {
    g_err[0] = 0;
    if (!q || !k || !v || !o || !scores || !ws)
        return fail(MINIKV_ERR_INVALID_ARG, "select_prefill: null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(ws))
        return fail(MINIKV_ERR_INVALID_ARG, "select_prefill: pointers must be 16-byte aligned");
    if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || Hq % Hkv)
        return fail(MINIKV_ERR_INVALID_ARG, "select_prefill: B=%d Hq=%d Hkv=%d T=%d", B, Hq, Hkv, T);
    if (D != kD) return fail(MINIKV_ERR_UNSUPPORTED, "select_prefill: D=%d (only 128)", D);
    if (!(sm_scale > 0.f) || !(sm_scale < INFINITY))
        return fail(MINIKV_ERR_INVALID_ARG, "select_prefill: sm_scale must be positive and finite");
    if (W < 1 || W > T) return fail(MINIKV_ERR_INVALID_ARG, "select_prefill: W=%d must be in [1, T=%d]", W, T);
    if ((Hq / Hkv) * W > 512) return fail(MINIKV_ERR_UNSUPPORTED, "select_prefill: (Hq/Hkv)*W above 512");
    if ((size_t)B * Hq > 65535 || (size_t)B * Hkv > 65535)
        return fail(MINIKV_ERR_UNSUPPORTED, "select_prefill: B*Hq above 65535");
    const size_t need = prefill_workspace_bytes(B, Hq, W);
    if (ws_bytes < need)
        return fail(MINIKV_ERR_INVALID_ARG, "select_prefill: workspace of %zu bytes needed, %zu given", need, ws_bytes);
    return prefill_launch(q, k, v, B, Hq, Hkv, T, W, sm_scale, o, scores, ws, static_cast<cudaStream_t>(stream));
}

int minikv_select_prefill_status(const void *ws, size_t ws_bytes, int B, int Hq, int W, void *stream,
                                 unsigned *status) {
    g_err[0] = 0;
    if (!ws || !status) return fail(MINIKV_ERR_INVALID_ARG, "select_prefill_status: null pointer");
    if (B < 1 || Hq < 1 || W < 1) return fail(MINIKV_ERR_INVALID_ARG, "select_prefill_status: B=%d Hq=%d W=%d", B, Hq, W);
    if (ws_bytes < prefill_workspace_bytes(B, Hq, W))
        return fail(MINIKV_ERR_INVALID_ARG, "select_prefill_status: workspace of %zu bytes is smaller than the call's",
                    ws_bytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const char *word = static_cast<const char *>(ws) + prefill_lse_bytes(B, Hq, W);
    cudaError_t e = cudaMemcpyAsync(status, word, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(MINIKV_ERR_CUDA, "select_prefill_status: %s", cudaGetErrorString(e));
    return MINIKV_OK;
}

int minikv_topk_evict(const float *scores, const uint16_t *k, const uint16_t *v, int B, int Hkv, int T, int D, int W,
                      int keep, int32_t *idx, uint16_t *k_kept, uint16_t *v_kept, void *ws, size_t ws_bytes,
                      void *stream) {
    g_err[0] = 0;
    (void)ws;
    (void)ws_bytes;
    if (!scores || !k || !v || !idx || !k_kept || !v_kept)
        return fail(MINIKV_ERR_INVALID_ARG, "topk_evict: null pointer");
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_kept) || !aligned16(v_kept))
        return fail(MINIKV_ERR_INVALID_ARG, "topk_evict: K/V pointers must be 16-byte aligned");
    if (B < 1 || Hkv < 1 || T < 1 || W < 0 || keep < 1)
        return fail(MINIKV_ERR_INVALID_ARG, "topk_evict: B=%d Hkv=%d T=%d W=%d keep=%d", B, Hkv, T, W, keep);
    if (D != kD) return fail(MINIKV_ERR_UNSUPPORTED, "topk_evict: D=%d (only 128)", D);
    if (keep < T && W > keep)
        return fail(MINIKV_ERR_INVALID_ARG, "topk_evict: window W=%d above the budget keep=%d", W, keep);
    if ((size_t)B * Hkv > 65535) return fail(MINIKV_ERR_UNSUPPORTED, "topk_evict: B*Hkv above 65535");
    return topk_launch(scores, k, v, B, Hkv, T, W, keep, idx, k_kept, v_kept, static_cast<cudaStream_t>(stream));
}

// shared by minikv_evict_pack (seq < 0: B prompts into every sequence) and
// minikv_evict_pack_seq (one prompt into sequence seq)
static int evict_pack_impl(const float *scores, const uint16_t *k, const uint16_t *v, int B, int Hkv, int T, int D,
                           int W, int keep, int32_t *idx, minikv_cache *c, int seq, void *stream) {
    g_err[0] = 0;
    int rc = check_cache(c);
    if (rc) return rc;
    if (!scores || !k || !v || !idx) return fail(MINIKV_ERR_INVALID_ARG, "evict_pack: null pointer");
    if (!aligned16(k) || !aligned16(v))
        return fail(MINIKV_ERR_INVALID_ARG, "evict_pack: K/V pointers must be 16-byte aligned");
    if (B < 1 || Hkv < 1 || T < 1 || W < 0 || keep < 1)
        return fail(MINIKV_ERR_INVALID_ARG, "evict_pack: B=%d Hkv=%d T=%d W=%d keep=%d", B, Hkv, T, W, keep);
    if (D != kD) return fail(MINIKV_ERR_UNSUPPORTED, "evict_pack: D=%d (only 128)", D);
    if (seq >= 0) {
        if (!c->seq && !c->dseq) return fail(MINIKV_ERR_INVALID_ARG, "evict_pack_seq: the cache is not ragged");
        if (seq >= c->B) return fail(MINIKV_ERR_INVALID_ARG, "evict_pack_seq: sequence %d of %d", seq, c->B);
        if (Hkv != c->Hkv)
            return fail(MINIKV_ERR_INVALID_ARG, "evict_pack_seq: Hkv=%d but the cache has Hkv=%d", Hkv, c->Hkv);
    } else if (B != c->B || Hkv != c->Hkv) {
        return fail(MINIKV_ERR_INVALID_ARG, "evict_pack: B=%d Hkv=%d but the cache has B=%d Hkv=%d", B, Hkv, c->B,
                    c->Hkv);
    }
    if (keep < T && W > keep)
        return fail(MINIKV_ERR_INVALID_ARG, "evict_pack: window W=%d above the budget keep=%d", W, keep);
    if ((size_t)B * Hkv > 65535) return fail(MINIKV_ERR_UNSUPPORTED, "evict_pack: B*Hkv above 65535");
    const int n = keep < T ? keep : T;
    int n_q = 0;
    if (n >= c->R) n_q = n - (c->R + (n - c->R) % c->G);
    if (n_q > c->cap) return fail(MINIKV_ERR_CAPACITY, "evict_pack: %d packed tokens exceed cap=%d", n_q, c->cap);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    rc = select_launch(scores, B, Hkv, T, W, keep, idx, s);
    if (rc) return rc;
    return pack_launch(c, k, v, n, s, idx, T, seq);
}

int minikv_evict_pack(const float *scores, const uint16_t *k, const uint16_t *v, int B, int Hkv, int T, int D, int W,
                      int keep, int32_t *idx, minikv_cache *c, void *stream) {
    return evict_pack_impl(scores, k, v, B, Hkv, T, D, W, keep, idx, c, -1, stream);
}

int minikv_evict_pack_seq(const float *scores, const uint16_t *k, const uint16_t *v, int Hkv, int T, int D, int W,
                          int keep, int32_t *idx, minikv_cache *c, int b, void *stream) {
    if (b < 0) {
        g_err[0] = 0;
        return fail(MINIKV_ERR_INVALID_ARG, "evict_pack_seq: sequence %d", b);
    }
    return evict_pack_impl(scores, k, v, 1, Hkv, T, D, W, keep, idx, c, b, stream);
}

int minikv_decode_attn(minikv_cache *c, const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new, int Hq,
                       float sm_scale, uint16_t *out, void *ws, size_t ws_bytes, void *stream) {
    int rc = decode_validate(c, q, k_new, v_new, Hq, out);
    if (rc) return rc;
    if (!ws) return fail(MINIKV_ERR_INVALID_ARG, "decode_attn: null workspace");
    if (!aligned16(ws)) return fail(MINIKV_ERR_INVALID_ARG, "decode_attn: workspace must be 16-byte aligned");
    return decode_launch(c, q, k_new, v_new, Hq, sm_scale, out, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int minikv_decode_attn_mass(minikv_cache *c, const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new, int Hq,
                            float sm_scale, uint16_t *out, float *mass, void *ws, size_t ws_bytes, void *stream) {
    int rc = decode_validate(c, q, k_new, v_new, Hq, out);
    if (rc) return rc;
    if (!ws || !mass) return fail(MINIKV_ERR_INVALID_ARG, "decode_attn_mass: null workspace or mass");
    if (!aligned16(ws)) return fail(MINIKV_ERR_INVALID_ARG, "decode_attn_mass: workspace must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(mass) & 3u)
        return fail(MINIKV_ERR_INVALID_ARG, "decode_attn_mass: mass must be 4-byte aligned");
    return decode_launch(c, q, k_new, v_new, Hq, sm_scale, out, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                         mass);
}

int minikv_set_deterministic(int on) {
    decode_set_deterministic(on);
    return MINIKV_OK;
}

int minikv_decode_plan(const minikv_cache *c, int *ctas, int *boundary_weight, int *first_items, int n_first) {
    const int rc = check_cache(c);
    if (rc) return rc;
    if (!ctas || !boundary_weight || n_first < 0 || (n_first > 0 && !first_items))
        return fail(MINIKV_ERR_INVALID_ARG, "decode_plan: null output or negative n_first");
    if ((size_t)c->B * c->Hkv > 65535) return fail(MINIKV_ERR_UNSUPPORTED, "decode_plan: B*Hkv above 65535");
    if ((size_t)c->B * c->Hkv * (c->cap / 32 + (c->R + c->G + 4) / 5) >= (1u << 31))
        return fail(MINIKV_ERR_UNSUPPORTED, "decode_plan: B*Hkv*(cap/32 + (R+G)/5) must stay below 2^31");
    return decode_plan_info(c, ctas, boundary_weight, n_first > 0 ? first_items : nullptr, n_first);
}

size_t minikv_workspace_size(int op, int B, int Hq, int Hkv, int T, int D, int W) {
    (void)D;
    switch (op) {
        case MINIKV_OP_SELECT_PREFILL: return prefill_workspace_bytes(B, Hq, W);
        case MINIKV_OP_TOPK_EVICT: return 0;
        case MINIKV_OP_DECODE_ATTN: return decode_workspace_bytes(B, Hkv, T);
        case MINIKV_OP_DECODE_ATTN_MASS:
            if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv || T < 0) return 0;
            return decode_mass_workspace_bytes(B, Hq, Hkv, T);
        default: return 0;
    }
}

}  // extern "C"
