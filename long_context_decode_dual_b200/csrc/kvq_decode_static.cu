// kvq_decode_attn_static: the decode entry point for callers that cannot
// allocate device memory when they call it.
//
// Some callers cannot hand the library a workspace: a plugin running inside a
// host inference engine that owns every device allocation and exposes no
// scratch buffer, or a latency-critical decode loop that must not call
// cudaMalloc (which can synchronise the device) on its hot path.  For them
// this entry point takes the split partials that kvq_decode_attn keeps in its
// caller-provided workspace from a fixed array in device memory instead.
//
// The array is a file-scope __device__ variable of kStaticScratchBytes.  Every
// GPU that loads this library keeps it for the life of the process.  Host code
// cannot pass the variable's name to a kernel (on the host the name is a
// stand-in, not a device address), so the device address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the
// first call made on that device, and cached.
#include <mutex>

#include "kvq_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;   // 4 MiB
constexpr int kMaxDevices = 128;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once).
int static_scratch_address(void **addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVQ_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return KVQ_OK;
}

}  // namespace

extern "C" {

size_t kvq_decode_static_scratch_bytes(void) { return kStaticScratchBytes; }

int kvq_decode_attn_static(const kvq_cache *cache, int n_q_heads, const int32_t *idx,
                           const float *qsel, const float *qgsum, int k, float *out,
                           kvq_stream_t stream) {
    const size_t need = kvq_decode_workspace(cache, n_q_heads, k);
    if (need > kStaticScratchBytes) return KVQ_ERR_WORKSPACE;
    void *scratch = nullptr;
    const int st = static_scratch_address(&scratch);
    if (st != KVQ_OK) return st;
    // nothing in the partials needs to start at zero: every split writes its
    // running max, sum and output before the merge reads them
    return kvq_decode_attn(cache, n_q_heads, idx, qsel, qgsum, k, out, scratch, kStaticScratchBytes,
                           stream);
}

}  // extern "C"
