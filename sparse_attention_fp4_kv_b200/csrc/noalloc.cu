// csa2_decode_stack_noalloc: the decode step of csa2_decode_stack for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc. Code that runs while a stream is being
// captured into a CUDA graph may not allocate. A plugin host may hand a kernel
// only its input and output tensors and keep every allocation to itself. A
// latency-critical serving loop cannot afford the device-wide synchronisation
// that cudaMalloc/cudaFree may cause. This entry point takes the same arguments
// as csa2_decode_stack except the workspace. Its scratch space (token scores,
// block scores, block counts, pooled scores and positions) lives in one
// file-scope device array of CSA2_NOALLOC_SCRATCH_BYTES, which every GPU that
// loads the library holds until the process exits.
//
// The host needs the array's device address. The first call on each device,
// with that device current, looks it up once with cudaGetSymbolAddress and
// caches it for the life of the process (a cudaDeviceReset destroys the context
// the cached address belongs to; the entry point must not be called on that
// device afterwards). Make that first call before any stream capture. Every call shares
// the one array: calls that overlap on the GPU (different streams, or
// concurrent host threads on the same device) race on it. Nothing in it has to
// start at zero: each call writes every scratch byte it reads before reading it.
#include <mutex>

#include "attention.cuh"

static __device__ __align__(256) uint8_t g_noalloc_scratch[CSA2_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device (looked up once
// per device), or nullptr on failure.
void *scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" int csa2_decode_stack_noalloc(const csa2_layer *layers, int n_layers,
                                         const void *kv_new_bf16, const int8_t *k_idx,
                                         const float *k_scale, uint8_t *kv_fp4, uint8_t *kv_sf,
                                         int64_t cap, const int64_t *ctx_len,
                                         const int64_t *swa_pos0, int swa_rows, int B, int Hq,
                                         int C, int H, int D, float softmax_scale, int32_t *pool,
                                         int pool_ready, void *stream) {
    if (B < 1 || cap < 1) return CSA2_ERR_SHAPE;
    const size_t need = csa2_decode_stack_workspace_size(B, Hq, C, H, D, cap);
    if (need > (size_t)CSA2_NOALLOC_SCRATCH_BYTES) return CSA2_ERR_WORKSPACE;
    void *scratch = scratch_address();
    if (scratch == nullptr) return CSA2_ERR_CUDA;
    return csa2_decode_stack(layers, n_layers, kv_new_bf16, k_idx, k_scale, kv_fp4, kv_sf, cap,
                             ctx_len, swa_pos0, swa_rows, B, Hq, C, H, D, softmax_scale, pool,
                             pool_ready, nullptr, scratch, (size_t)CSA2_NOALLOC_SCRATCH_BYTES,
                             stream);
}
