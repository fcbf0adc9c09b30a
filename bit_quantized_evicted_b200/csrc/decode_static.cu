// minikv_decode_attn_static: the decode step for callers that may not
// allocate device memory.
//
// minikv_decode_attn needs a caller-supplied workspace for its split-KV
// partial results and arrival counters.  Some callers cannot provide one: a
// host whose device memory is entirely planned by its own allocator or memory
// pool (a cudaMalloc behind its back breaks its accounting and budget), or a
// latency-critical loop where cudaMalloc is not allowed because it can
// synchronize the device.  This entry point runs the same decode kernel with
// its scratch taken from a fixed array that lives in this library's module:
// `g_decode_scratch`, kStaticScratchBytes (8 MiB) per GPU, held by every GPU
// that loads the library until the process exits.
//
// Set-up: the first call on a device looks up the device address of the array
// (cudaGetSymbolAddress, with that device current) and keeps it; make that
// first call before any stream capture.  Every call shares the one array and
// leaves its last contents there, so calls whose GPU work overlaps (two
// streams, two host threads on one device) race on it; each call first clears
// the arrival counters, which must start at zero.  No call allocates or frees
// device memory.
#include <mutex>

#include "common.cuh"

namespace minikv {

int decode_launch(minikv_cache *c, const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new, int Hq,
                  float sm_scale, uint16_t *out, void *ws, size_t ws_bytes, cudaStream_t stream,
                  float *mass = nullptr);
int decode_validate(minikv_cache *c, const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new, int Hq,
                    const uint16_t *out);
size_t decode_counter_bytes(int B, int Hkv);
size_t decode_call_workspace_bytes(const minikv_cache *c);

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once).
// The work is queued on `stream`, so the stream must belong to that device:
// otherwise the kernel would clear and use another GPU's copy of the array.
int scratch_address(cudaStream_t stream, void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(MINIKV_ERR_CUDA, "decode_attn_static: cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(MINIKV_ERR_UNSUPPORTED, "decode_attn_static: device %d", dev);
    int sdev = -1;
    e = cudaStreamGetDevice(stream, &sdev);
    if (e != cudaSuccess)
        return fail(MINIKV_ERR_INVALID_ARG, "decode_attn_static: cudaStreamGetDevice: %s", cudaGetErrorString(e));
    if (sdev != dev)
        return fail(MINIKV_ERR_INVALID_ARG, "decode_attn_static: the stream belongs to device %d, the current device is %d",
                    sdev, dev);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || !p)
            return fail(MINIKV_ERR_CUDA, "decode_attn_static: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MINIKV_OK;
}

}  // namespace
}  // namespace minikv

using namespace minikv;

extern "C" int minikv_decode_attn_static(minikv_cache *c, const uint16_t *q, const uint16_t *k_new,
                                         const uint16_t *v_new, int Hq, float sm_scale, uint16_t *out,
                                         void *stream) {
    int rc = decode_validate(c, q, k_new, v_new, Hq, out);
    if (rc) return rc;
    const size_t need = decode_call_workspace_bytes(c);
    if (need > kStaticScratchBytes)
        return fail(MINIKV_ERR_UNSUPPORTED,
                    "decode_attn_static: this step needs %zu bytes of scratch but the static buffer holds %zu; "
                    "use minikv_decode_attn with a caller workspace",
                    need, kStaticScratchBytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void *scratch = nullptr;
    rc = scratch_address(s, &scratch);
    if (rc) return rc;
    cudaError_t e = cudaMemsetAsync(scratch, 0, decode_counter_bytes(c->B, c->Hkv), s);
    if (e != cudaSuccess)
        return fail(MINIKV_ERR_CUDA, "decode_attn_static: clearing counters: %s", cudaGetErrorString(e));
    return decode_launch(c, q, k_new, v_new, Hq, sm_scale, out, scratch, kStaticScratchBytes, s);
}
