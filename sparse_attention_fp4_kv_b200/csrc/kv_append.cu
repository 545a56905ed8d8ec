// FP4 main-KV append: quantize-and-pack new bf16 rows into the cache.
//
// "DeepSeek V4.1 Flash KV Cache: 890 Bytes per Token Explained" (FP4 section)
// and "DeepSeek-V4.1-Flash: 890 Bytes Per Token, 437x Smaller KV Cache" (FP4
// KV Quantization section): E2M1 elements, one E4M3 scale per 16 channels,
// the NVFP4 scheme without its global scale.
//
// One thread per 16-channel group: two 16-byte loads of bf16, the group's
// amax, the scale amax/6 rounded to E4M3 (PTX cvt, RNE + saturation), then 16
// IEEE fp32 divisions by the decoded scale and eight E2M1 pair conversions.
// A warp covers 512 contiguous channels, so loads (32 B per lane), packed
// stores (8 B per lane) and scale stores (1 B per lane) are all coalesced.
// The cost is negligible in decode (one row per sequence) and a few MB of
// traffic in chunked prefill.
#include "common.cuh"

namespace csa2 {

// 16-channel group gid of the B x n_new new rows.
__device__ __forceinline__ void kv_append_group(const uint16_t *__restrict__ kv, int B, int n_new,
                                                int C, const int64_t *__restrict__ start_pos,
                                                int64_t pos_offset, int64_t cap,
                                                uint8_t *__restrict__ fp4, uint8_t *__restrict__ sf,
                                                int64_t gid) {
    const int G = C / 16;
    const int64_t total = (int64_t)B * n_new * G;
    if (gid >= total) return;
    const int g = (int)(gid % G);
    const int64_t row = gid / G;  // b * n_new + i
    const int i = (int)(row % n_new);
    const int b = (int)(row / n_new);
    const int64_t pos = start_pos[b] + pos_offset + i;
    if (pos < 0 || pos >= cap) return;

    const uint4 *src = reinterpret_cast<const uint4 *>(kv + row * C + (int64_t)g * 16);
    const uint4 a = src[0], c = src[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
    float x[16];
#pragma unroll
    for (int j = 0; j < 8; j++) {
        x[2 * j] = bf16_lo(w[j]);
        x[2 * j + 1] = bf16_hi(w[j]);
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; j++) amax = fmaxf(amax, fabsf(x[j]));

    const uint32_t scode = f32_to_e4m3_satfinite(__fdiv_rn(amax, 6.0f));
    const float s = e4m3_to_f32(scode);
    uint32_t lo = 0, hi = 0;
    if (s != 0.0f) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; j++) v[j] = __fdiv_rn(x[j], s);
        lo = f32x8_to_e2m1x8(v);
        hi = f32x8_to_e2m1x8(v + 8);
    }
    const int64_t cell = (int64_t)b * cap + pos;
    *reinterpret_cast<uint2 *>(fp4 + cell * (C / 2) + (int64_t)g * 8) = make_uint2(lo, hi);
    sf[cell * G + g] = (uint8_t)scode;
}

__global__ void __launch_bounds__(256) kv_append_fp4_kernel(
    const uint16_t *__restrict__ kv, int B, int n_new, int C, const int64_t *__restrict__ start_pos,
    int64_t pos_offset, int64_t cap, uint8_t *__restrict__ fp4, uint8_t *__restrict__ sf) {
    grid_dep_wait();
    grid_dep_launch();
    kv_append_group(kv, B, n_new, C, start_pos, pos_offset, cap, fp4, sf,
                    (int64_t)blockIdx.x * blockDim.x + threadIdx.x);
}

// First kernel of a decode step: the new token's row of every sequence (at
// position ctx_len - 1, when kv is given) and the zeroing of the step's two
// workspace regions that must start at zero (z0 [n0], z1 [n1] 16-byte words).
// A kernel instead of memsets keeps the step one chain of dependent launches.
__global__ void __launch_bounds__(256) decode_step_begin_kernel(
    const uint16_t *__restrict__ kv, int B, int C, const int64_t *__restrict__ ctx_len, int64_t cap,
    uint8_t *__restrict__ fp4, uint8_t *__restrict__ sf, uint4 *z0, int64_t n0, uint4 *z1, int64_t n1) {
    grid_dep_wait();
    grid_dep_launch();
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    if (kv)
        for (int64_t g = gid; g < (int64_t)B * (C / 16); g += stride)
            kv_append_group(kv, B, 1, C, ctx_len, -1, cap, fp4, sf, g);
    for (int64_t i = gid; i < n0; i += stride) z0[i] = make_uint4(0, 0, 0, 0);
    for (int64_t i = gid; i < n1; i += stride) z1[i] = make_uint4(0, 0, 0, 0);
}

// MXFP4 variant: one thread per 32-channel block. The shared exponent is the
// exponent of the block's amax minus 2 (the largest E2M1 exponent), clamped to
// the E8M0 range: read straight from the fp32 exponent field, so an all-zero or
// subnormal amax gives 2^-127. Elements are x * 2^-e, an exact scaling since
// the result stays below 8, then the same E2M1 pair conversion.
__global__ void __launch_bounds__(256) kv_append_mxfp4_kernel(
    const uint16_t *__restrict__ kv, int B, int n_new, int C, const int64_t *__restrict__ start_pos,
    int64_t pos_offset, int64_t cap, uint8_t *__restrict__ fp4, uint8_t *__restrict__ sf) {
    grid_dep_wait();
    grid_dep_launch();
    const int G = C / 32;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = (int64_t)B * n_new * G;
    if (gid >= total) return;
    const int g = (int)(gid % G);
    const int64_t row = gid / G;
    const int i = (int)(row % n_new);
    const int b = (int)(row / n_new);
    const int64_t pos = start_pos[b] + pos_offset + i;
    if (pos < 0 || pos >= cap) return;

    const uint4 *src = reinterpret_cast<const uint4 *>(kv + row * C + (int64_t)g * 32);
    float x[32];
#pragma unroll
    for (int q = 0; q < 4; q++) {
        const uint4 a = src[q];
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            x[8 * q + 2 * j] = bf16_lo(w[j]);
            x[8 * q + 2 * j + 1] = bf16_hi(w[j]);
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; j++) amax = fmaxf(amax, fabsf(x[j]));
    const int E = (int)((__float_as_uint(amax) >> 23) & 0xFF);  // 0 for zero / subnormal
    int e = E == 0 ? -127 : E - 129;
    e = e < -127 ? -127 : e;
    // 2^-e as an fp32: e lies in [-127, 126], so 2^-e is a normal number
    // (2^-126 .. 2^127)
    const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; j++) v[j] = x[j] * inv;
    const int64_t cell = (int64_t)b * cap + pos;
    uint2 *dst = reinterpret_cast<uint2 *>(fp4 + cell * (C / 2) + (int64_t)g * 16);
    dst[0] = make_uint2(f32x8_to_e2m1x8(v), f32x8_to_e2m1x8(v + 8));
    dst[1] = make_uint2(f32x8_to_e2m1x8(v + 16), f32x8_to_e2m1x8(v + 24));
    sf[cell * G + g] = (uint8_t)(e + 127);
}

int launch_kv_append(const uint16_t *kv, int B, int n_new, int C, const int64_t *pos_base,
                     int64_t pos_offset, int64_t cap, uint8_t *fp4, uint8_t *sf, cudaStream_t s,
                     bool pdl) {
    const int64_t total = (int64_t)B * n_new * (C / 16);
    if (total == 0) return CSA2_OK;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    if (blocks > INT32_MAX) return CSA2_ERR_SHAPE;
    return launch_kernel(pdl, kv_append_fp4_kernel, dim3((unsigned)blocks), dim3(threads), 0, s, kv,
                         B, n_new, C, pos_base, pos_offset, cap, fp4, sf);
}

int launch_decode_step_begin(const uint16_t *kv, int B, int C, const int64_t *ctx_len, int64_t cap,
                             uint8_t *fp4, uint8_t *sf, void *z0, size_t z0_bytes, void *z1,
                             size_t z1_bytes, cudaStream_t s) {
    const int64_t n0 = (int64_t)(z0_bytes / 16), n1 = (int64_t)(z1_bytes / 16);
    int64_t work = kv ? (int64_t)B * (C / 16) : 0;
    if (n0 + n1 > work) work = n0 + n1;
    int64_t blocks = (work + 256 * 4 - 1) / (256 * 4);  // about 4 items per thread
    if (blocks < 1) blocks = 1;
    if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
    return launch_kernel(true, decode_step_begin_kernel, dim3((unsigned)blocks), dim3(256), 0, s, kv, B,
                         C, ctx_len, cap, fp4, sf, static_cast<uint4 *>(z0), n0,
                         static_cast<uint4 *>(z1), n1);
}

}  // namespace csa2

extern "C" int csa2_kv_append_fp4(const void *kv_bf16, int B, int n_new, int C,
                                  const int64_t *start_pos, int64_t cap, uint8_t *kv_fp4,
                                  uint8_t *kv_sf, void *stream) {
    using namespace csa2;
    if (!kv_bf16 || !start_pos || !kv_fp4 || !kv_sf) return CSA2_ERR_NULL;
    if (B < 0 || n_new < 0 || cap < 0 || C < 16 || C > 8192 || C % 16) return CSA2_ERR_SHAPE;
    if (!aligned(kv_bf16, 16) || !aligned(kv_fp4, 8)) return CSA2_ERR_ALIGN;
    return launch_kv_append((const uint16_t *)kv_bf16, B, n_new, C, start_pos, 0, cap, kv_fp4,
                            kv_sf, (cudaStream_t)stream);
}

extern "C" int csa2_kv_append_mxfp4(const void *kv_bf16, int B, int n_new, int C,
                                    const int64_t *start_pos, int64_t cap, uint8_t *kv_fp4,
                                    uint8_t *kv_sf, void *stream) {
    using namespace csa2;
    if (!kv_bf16 || !start_pos || !kv_fp4 || !kv_sf) return CSA2_ERR_NULL;
    if (B < 0 || n_new < 0 || cap < 0 || C < 32 || C > 8192 || C % 32) return CSA2_ERR_SHAPE;
    if (!aligned(kv_bf16, 16) || !aligned(kv_fp4, 8)) return CSA2_ERR_ALIGN;
    const int64_t total = (int64_t)B * n_new * (C / 32);
    if (total == 0) return CSA2_OK;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    if (blocks > INT32_MAX) return CSA2_ERR_SHAPE;
    return launch_kernel(false, kv_append_mxfp4_kernel, dim3((unsigned)blocks), dim3(threads), 0,
                         (cudaStream_t)stream, (const uint16_t *)kv_bf16, B, n_new, C, start_pos,
                         (int64_t)0, cap, kv_fp4, kv_sf);
}
