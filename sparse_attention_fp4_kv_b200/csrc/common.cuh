// Shared helpers of the libcsa2 CUDA sources (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "csa2.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libcsa2 is written for sm_100a (B200) only"
#endif

namespace csa2 {

constexpr int kPoolBlocks = CSA2_POOL_BLOCKS;
constexpr int kBlockTokens = CSA2_BLOCK_TOKENS;
constexpr int kTopK = CSA2_TOPK;
constexpr int kWarp = 32;

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int launch_status() {
    return cudaGetLastError() == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

// ---------------------------------------------------------------- per-device set-up
// Function attributes (the dynamic shared-memory limit, the carveout) and
// occupancy figures belong to one device. Launchers keep their one-time set-up
// in a PerDevice table indexed by the current device ordinal, so a process that
// drives several GPUs sets each one up once, and host threads may race to the
// first call safely.
constexpr int kMaxDevices = 64;

class PerDevice {
  public:
    // The value for the current device; fn() computes it the first time and
    // returns a value >= 0, or < 0 on failure (then nothing is cached and the
    // next call tries again). Devices past kMaxDevices are never cached.
    template <class F>
    int get(F &&fn) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return fn();
        int v = value_[dev].load(std::memory_order_acquire);
        if (v > 0) return v - 1;
        std::lock_guard<std::mutex> lock(mutex_);
        v = value_[dev].load(std::memory_order_relaxed);
        if (v > 0) return v - 1;
        const int r = fn();
        if (r >= 0) value_[dev].store(r + 1, std::memory_order_release);
        return r;
    }

  private:
    std::mutex mutex_;
    std::atomic<int> value_[kMaxDevices] = {};  // value + 1; 0 = not yet computed
};

// Sets the dynamic shared-memory limit of `kernel` on the current device once.
template <typename K>
inline bool set_smem_limit_once(PerDevice &done, K kernel, size_t bytes) {
    return done.get([&] {
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) ==
                       cudaSuccess
                   ? 1
                   : -1;
    }) >= 0;
}

// ---------------------------------------------------------------- dependent launches
// Kernels of one decode step may be launched with programmatic stream
// serialization: the next kernel's CTAs can be scheduled while the previous
// kernel on the stream is still running. Every kernel therefore calls
// grid_dep_wait() before its first access to memory that the previous kernel
// may read or write (the wait returns once that grid has completed and its
// writes are visible), and grid_dep_launch() right after it, so that a
// kernel which starts early can rely on everything launched two or more
// kernels before it being complete. Both are no-ops in a kernel launched
// without the attribute.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch `kernel`, with programmatic stream serialization when pdl is true.
template <typename... KArgs, typename... Args>
inline int launch_kernel(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                         cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess)
        return CSA2_ERR_CUDA;
    return launch_status();
}

// Reads a device flag of the library (an int __device__ variable of the
// calling translation unit), resetting it when clear; -1 if it cannot be read.
template <typename T>
inline int read_device_flag(T &symbol, bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, symbol, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int z = 0;
        if (cudaMemcpyToSymbol(symbol, &z, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}
// The bounded-wait flags of the kernels that wait on the device.
int attn_tc_wait_flag(bool clear);
int attn_rows_wait_flag(bool clear);
int index_mma_wait_flag(bool clear);

// Streaming multiprocessors of the current device (148 on B200 if the query fails).
inline int num_sms() {
    static PerDevice cache;
    return cache.get([] {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        return n;
    });
}

// ---------------------------------------------------------------- bf16 / fp8 / fp4
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Prefetch of a contiguous global range into L2 (16-byte aligned, size a
// multiple of 16); no data reaches the issuing CTA.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// E4M3 code -> fp32 from the format definition (1 sign, 4 exponent bits with
// bias 7, 3 mantissa bits; exponent field 0 is subnormal m * 2^-9). Exact.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t e = (code >> 3) & 0xF, m = code & 7;
    float mag = (e == 0) ? (float)m * 0.001953125f                     // m * 2^-9
                         : __uint_as_float(((e + 120u) << 23) | (m << 20));  // 2^(e-7)(1+m/8)
    return (code & 0x80) ? -mag : mag;
}

// E2M1 magnitude code (3 bits) -> fp32: 0, .5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ float e2m1_mag(uint32_t c3) {
    uint32_t e = c3 >> 1, m = c3 & 1;
    return (e == 0) ? 0.5f * (float)m : __uint_as_float(((e + 126u) << 23) | (m << 22));
}
__device__ __forceinline__ float e2m1_to_f32(uint32_t c4) {
    float v = e2m1_mag(c4 & 7);
    return (c4 & 8) ? -v : v;
}

// E8M0 scale (MXFP4 variant): code e is 2^(e - 127), 255 is NaN; code 0 is the
// fp32 subnormal 2^-127.
__device__ __forceinline__ float e8m0_to_f32(uint32_t code) {
    if (code == 255u) return __uint_as_float(0x7FC00000u);
    return code == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(code << 23);
}
// Scale of 16-channel group g of a row whose scale bytes start at sf: E4M3
// per 16 channels, or (mx) E8M0 per 32 channels.
__device__ __forceinline__ float kv_group_scale(const uint8_t *sf, int g, bool mx) {
    return mx ? e8m0_to_f32(sf[g >> 1]) : e4m3_to_f32(sf[g]);
}

__device__ __forceinline__ uint32_t f32_to_e4m3_satfinite(float x) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
    return r & 0xFF;
}

// Eight fp32 values -> eight E2M1 codes packed in a 32-bit word, value j in
// nibble j (round-to-nearest-even, saturation to +-6; PTX cvt places its
// second source in the low nibble of each byte).
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float *v) {
    uint32_t r;
    asm("{\n"
        ".reg .b8 b0, b1, b2, b3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
        "mov.b32 %0, {b0, b1, b2, b3};\n"
        "}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// ---------------------------------------------------------------- ordering keys
// fp32 -> uint32 whose unsigned order is the float order (-0 folded onto +0).
__device__ __forceinline__ uint32_t f32_order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 64-bit rank key: higher key = better candidate (score desc, position asc).
__device__ __forceinline__ uint64_t rank_key(float score, int32_t pos) {
    return ((uint64_t)f32_order_key(score) << 32) | (uint32_t)(~(uint32_t)pos);
}
__device__ __forceinline__ int32_t rank_key_pos(uint64_t key) { return (int32_t)(~(uint32_t)key); }

// ---------------------------------------------------------------- loads
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Visible length of query (b, i): the whole context in decode, causal in prefill.
__device__ __forceinline__ int64_t visible_len(const int64_t *ctx_len, const int64_t *q_pos, int b,
                                               int i, int Nq) {
    int64_t v = ctx_len[b];
    if (q_pos) {
        int64_t p = q_pos[(int64_t)b * Nq + i] + 1;
        v = p < v ? p : v;
    }
    return v < 0 ? 0 : v;
}

// FP4 append with positions pos_base[b] + pos_offset + i (kv_append.cu).
int launch_kv_append(const uint16_t *kv, int B, int n_new, int C, const int64_t *pos_base,
                     int64_t pos_offset, int64_t cap, uint8_t *fp4, uint8_t *sf, cudaStream_t s,
                     bool pdl = false);

// First-digit histogram bin of a score (top 12 bits of its order-preserving
// key), shared by the score producers and the histogram-fed top-k.
constexpr int kHistBins = 4096;
__device__ __forceinline__ uint32_t hist_bin(float score) { return f32_order_key(score) >> 20; }

// Histogram-fed top-k (topk.cu): the workspace starts with hist[R][4096] and
// four counters per row, all zero before the producer runs. This launcher and
// the three score producers below serve the decode step only and launch with
// programmatic stream serialization.
size_t topk_hist_ws_bytes(int R, int k);
// The leading bytes of such a workspace (histogram rows and per-row counters)
// that must be zero before a producer adds to it.
size_t topk_hist_zero_bytes(int R);
// Pool and top tokens of the decode Full layer in one selection (topk.cu).
int launch_pool_and_tokens(const float *blk, const int32_t *n_blk, int R, int64_t nblk, int P,
                           int32_t *pool, void *ws, const float *tok, const int64_t *ctx_len,
                           int64_t cap, int ktop, int32_t *top, cudaStream_t s);
int launch_topk_from_hist(const float *score, const int32_t *cand_pos, const int32_t *n_valid,
                          int R, int64_t n, int k, int32_t *out, void *ws, cudaStream_t s);

// Score producers with an optional histogram output (indexer.cu).
int launch_index_full_hist(const int8_t *q_idx, const int8_t *k_idx, const float *k_scale,
                           const int64_t *ctx_len, int B, int H, int D, int64_t cap,
                           float *tok_score, float *blk_score, int32_t *n_blk, uint32_t *hist,
                           cudaStream_t s);
int launch_pool_gather_hist(const float *tok_score, const int32_t *pool, const int64_t *ctx_len,
                            int B, int P, int64_t cap, float *pool_score, int32_t *pool_pos,
                            uint32_t *hist, cudaStream_t s);
// The decode step's first kernel: the new rows' append (kv may be NULL) and the
// zeroing of two workspace regions (16-byte aligned, sizes multiples of 16).
int launch_decode_step_begin(const uint16_t *kv, int B, int C, const int64_t *ctx_len, int64_t cap,
                             uint8_t *fp4, uint8_t *sf, void *z0, size_t z0_bytes, void *z1,
                             size_t z1_bytes, cudaStream_t s);
int launch_reindex_hist(const int8_t *q_idx, const int8_t *k_idx, const float *k_scale,
                        const int32_t *pool, const int64_t *ctx_len, int B, int H, int D,
                        int64_t cap, int P, float *pool_score, int32_t *pool_pos, uint32_t *hist,
                        cudaStream_t s);

// Multi-query indexer scan on tensor cores (index_mma.cu).
bool index_mma_supported(int Nq, int HD, int64_t cap, int B);
int launch_index_mma(const int8_t *q, const int8_t *k, const float *kscale, const int64_t *ctx_len,
                     const int64_t *q_pos, int B, int Nq, int HD, int64_t cap, float *tok,
                     float *blk, int32_t *n_blk, cudaStream_t s);

}  // namespace csa2
