// Device-side error status: the kernels that wait on mbarriers bound every
// wait and, when a bound runs out, record it in a device flag and return
// (no trap, so the CUDA context stays usable). csa2_device_status reads the
// flags; csa2_selftest_wait_timeout exercises the path with a wait that no
// arrival completes.
#include "common.cuh"

namespace csa2 {

__device__ int g_selftest_error = 0;

__global__ void selftest_wait_kernel(uint64_t limit_ns, int *err) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // nobody arrives on the barrier: the wait below can only end by its bound
    uint64_t t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    bool done = false;
    do {
        uint32_t d;
        asm volatile(
            "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n"
            "selp.u32 %0, 1, 0, p;\n}"
            : "=r"(d)
            : "r"(b)
            : "memory");
        done = d != 0;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    } while (!done && t - t0 < limit_ns);
    if (!done && threadIdx.x == 0) {
        atomicExch(&g_selftest_error, 1);
        if (err) atomicExch(err, 1);
    }
}

}  // namespace csa2

using namespace csa2;

extern "C" int csa2_device_status(int clear) {
    if (cudaDeviceSynchronize() != cudaSuccess) return CSA2_ERR_CUDA;
    const int flags[4] = {attn_tc_wait_flag(clear != 0), attn_rows_wait_flag(clear != 0),
                          index_mma_wait_flag(clear != 0),
                          read_device_flag(g_selftest_error, clear != 0)};
    int any = 0;
    for (int f : flags) {
        if (f < 0) return CSA2_ERR_CUDA;
        any |= f;
    }
    return any ? CSA2_ERR_DEVICE_TIMEOUT : CSA2_OK;
}

extern "C" int csa2_selftest_wait_timeout(int limit_us, void *stream) {
    if (limit_us < 1 || limit_us > 1000000) return CSA2_ERR_RANGE;
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_us * 1000ull, nullptr);
    return launch_status();
}

extern "C" int csa2_selftest_workspace_timeout(int limit_us, void *ws, void *stream) {
    if (!ws) return CSA2_ERR_NULL;
    if (limit_us < 1 || limit_us > 1000000) return CSA2_ERR_RANGE;
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_us * 1000ull,
                                                               static_cast<int *>(ws));
    return launch_status();
}
