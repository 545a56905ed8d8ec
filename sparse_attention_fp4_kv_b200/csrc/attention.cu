// Sparse attention over the selected FP4 main-KV rows plus the sliding window.
//
// "890 bytes per token: how DeepSeek V4.1-Flash's KV cache works", mechanism
// 4: attention runs only over the candidates the indexer selected.
// "DeepSeek-V4.1-Flash: 890 Bytes Per Token, 437x Smaller KV Cache", CED and
// CSA2 sections: every layer computes its own main Q and SWA KV; the window is
// the last 128 tokens. The main KV is one shared head (K = V = the row), stored
// as E2M1 codes with one E4M3 scale per 16 channels; dequantization
// e2m1 * e4m3 is exact in fp32.
//
// General kernel: one CTA per (query, head). Warps compute one logit per key
// (lane = C/32 channels, dequantized in registers, fp32 dot, shuffle reduce),
// the CTA does the softmax in shared memory, and each thread then accumulates
// its channels over all keys. Used for shapes outside the tensor-core
// kernel's constraints (attention_tc.cu).
#include <cfloat>

#include "attention.cuh"

namespace csa2 {

__global__ void __launch_bounds__(256) attn_general_kernel(AttnArgs a) {
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ float sm[];
    const int C = a.C;
    float *qs = sm;            // [C]
    float *lg = sm + C;        // [K + n_win]
    __shared__ float red[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
    const int64_t bq = blockIdx.x / a.Hq;
    const int h = (int)(blockIdx.x % a.Hq);
    const int b = (int)(bq / a.Nq);

    AttnWindow w = attn_window(a, b, bq);
    const int nkeys = a.K + w.n;

    const uint16_t *q = reinterpret_cast<const uint16_t *>(a.q) + (bq * a.Hq + h) * (int64_t)C;
    for (int c = tid; c < C; c += blockDim.x) qs[c] = __uint_as_float((uint32_t)q[c] << 16);
    __syncthreads();

    const int CPL = C / 32;  // channels per lane
    for (int j = warp; j < nkeys; j += nwarp) {
        float dot = 0.0f;
        bool valid = true;
        if (j < a.K) {
            const int32_t pos = a.topk[bq * a.K + j];
            valid = pos >= 0 && pos < a.cap;
            if (valid) {
                const int64_t cell = (int64_t)b * a.cap + pos;
                const uint8_t *row = a.kv_fp4 + cell * (C / 2);
                const uint8_t *sfr = a.kv_sf + cell * (C / (a.mx ? 32 : 16));
                for (int u = 0; u < CPL; u += 2) {
                    const int c = lane * CPL + u;
                    const uint32_t byte = row[c / 2];
                    const float s = kv_group_scale(sfr, c / 16, a.mx);
                    dot += qs[c] * (e2m1_to_f32(byte & 0xF) * s);
                    dot += qs[c + 1] * (e2m1_to_f32(byte >> 4) * s);
                }
            }
        } else {
            const uint16_t *row = reinterpret_cast<const uint16_t *>(a.swa) +
                                  ((int64_t)b * a.swa_rows + w.row0 + (j - a.K)) * C;
            for (int u = 0; u < CPL; u++) {
                const int c = lane * CPL + u;
                dot += qs[c] * __uint_as_float((uint32_t)row[c] << 16);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        if (lane == 0) lg[j] = valid ? dot * a.scale : -INFINITY;
    }
    __syncthreads();

    // softmax statistics
    float m = -INFINITY;
    for (int j = tid; j < nkeys; j += blockDim.x) m = fmaxf(m, lg[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = -INFINITY;
    for (int w2 = 0; w2 < nwarp; w2++) m = fmaxf(m, red[w2]);
    __syncthreads();
    float z = 0.0f;
    for (int j = tid; j < nkeys; j += blockDim.x) {
        const float p = (lg[j] == -INFINITY) ? 0.0f : expf(lg[j] - m);
        lg[j] = p;
        z += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane == 0) red[warp] = z;
    __syncthreads();
    z = 0.0f;
    for (int w2 = 0; w2 < nwarp; w2++) z += red[w2];
    const float inv = z > 0.0f ? 1.0f / z : 0.0f;

    float *out = a.out + (bq * a.Hq + h) * (int64_t)C;
    for (int c = tid; c < C; c += blockDim.x) {
        float acc = 0.0f;
        for (int j = 0; j < a.K; j++) {
            const float p = lg[j];
            if (p == 0.0f) continue;
            const int64_t cell = (int64_t)b * a.cap + a.topk[bq * a.K + j];
            const uint32_t byte = a.kv_fp4[cell * (C / 2) + c / 2];
            const float v = e2m1_to_f32((c & 1) ? (byte >> 4) : (byte & 0xF)) *
                            kv_group_scale(a.kv_sf + cell * (C / (a.mx ? 32 : 16)), c / 16, a.mx);
            acc += p * v;
        }
        const uint16_t *swa = reinterpret_cast<const uint16_t *>(a.swa) +
                              ((int64_t)b * a.swa_rows + w.row0) * C;
        for (int j = 0; j < w.n; j++) {
            const float p = lg[a.K + j];
            acc += p * __uint_as_float((uint32_t)swa[(int64_t)j * C + c] << 16);
        }
        out[c] = acc * inv;
    }
}

int launch_attn_general(const AttnArgs &a, cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)a.C + a.K + a.n_win);
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(attn_general_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return CSA2_ERR_CUDA;
    }
    const int64_t grid = (int64_t)a.B * a.Nq * a.Hq;
    if (grid > INT32_MAX) return CSA2_ERR_SHAPE;
    return launch_kernel(a.pdl, attn_general_kernel, dim3((unsigned)grid), dim3(256), smem, s, a);
}

}  // namespace csa2

using namespace csa2;

extern "C" size_t csa2_sparse_attn_workspace_size(int B, int Nq, int Hq, int C, int K, int n_win) {
    return attn_workspace_bytes(B, Nq, Hq, C, K, n_win);
}

extern "C" int csa2_sparse_attn_decode(const void *q_bf16, const uint8_t *kv_fp4,
                                       const uint8_t *kv_sf, int64_t cap, const int32_t *topk,
                                       int K, const void *swa_bf16, const int64_t *swa_pos0,
                                       int swa_rows, const int64_t *q_pos, int n_win, int B,
                                       int Nq, int Hq, int C, float softmax_scale, float *out,
                                       void *ws, size_t ws_bytes, void *stream) {
    AttnArgs a{q_bf16, kv_fp4, kv_sf, cap, topk, K, swa_bf16, swa_pos0, swa_rows, q_pos,
               n_win, B, Nq, Hq, C, softmax_scale, out, ws, false, false};
    return attn_checked_launch(a, ws_bytes, (cudaStream_t)stream);
}

extern "C" int csa2_sparse_attn_decode_mxfp4(const void *q_bf16, const uint8_t *kv_fp4,
                                             const uint8_t *kv_sf, int64_t cap, const int32_t *topk,
                                             int K, const void *swa_bf16, const int64_t *swa_pos0,
                                             int swa_rows, const int64_t *q_pos, int n_win, int B,
                                             int Nq, int Hq, int C, float softmax_scale, float *out,
                                             void *ws, size_t ws_bytes, void *stream) {
    if (C % 32) return CSA2_ERR_SHAPE;
    AttnArgs a{q_bf16, kv_fp4, kv_sf, cap, topk, K, swa_bf16, swa_pos0, swa_rows, q_pos,
               n_win, B, Nq, Hq, C, softmax_scale, out, ws, false, false, true};
    return attn_checked_launch(a, ws_bytes, (cudaStream_t)stream);
}

namespace csa2 {

int attn_checked_launch(const AttnArgs &a, size_t ws_bytes, cudaStream_t s, bool validate_only) {
    if (!a.q || !a.kv_fp4 || !a.kv_sf || !a.out) return CSA2_ERR_NULL;
    if (a.K > 0 && !a.topk) return CSA2_ERR_NULL;
    if (a.n_win > 0 && a.swa_rows > 0 && (!a.swa || !a.swa_pos0)) return CSA2_ERR_NULL;
    if (!a.q_pos && !a.swa_pos0) return CSA2_ERR_NULL;
    if (a.B < 0 || a.Nq < 0 || a.cap < 1 || a.C < 32 || a.C > 1024 || a.C % 32 || a.Hq < 1 ||
        a.Hq > 256 || a.K < 0 || a.K > 4096 || a.n_win < 0 || a.n_win > 4096 || a.swa_rows < 0)
        return CSA2_ERR_SHAPE;
    if (!aligned(a.q, 16) || (a.swa && !aligned(a.swa, 16)) || !aligned(a.kv_fp4, 8))
        return CSA2_ERR_ALIGN;
    if (ws_bytes < attn_workspace_bytes(a.B, a.Nq, a.Hq, a.C, a.K, a.n_win))
        return CSA2_ERR_WORKSPACE;
    if ((int64_t)a.B * a.Nq == 0 || validate_only) return CSA2_OK;
    return launch_attn(a, s);
}

// The tensor-core kernel exchanges per-CTA partial results through the
// workspace; the general kernel needs none. The size covers the tensor-core
// path whenever its shape constraints could hold.
size_t attn_workspace_bytes(int B, int Nq, int Hq, int C, int K, int n_win) {
    if (C == 512 && Hq == 64 && K > 0 && K <= 640)
        return attn_tc_workspace_bytes(B, Nq);
    return 0;
}

// Tensor-core kernels where their shape constraints hold (64 heads, 512
// channels): one CTA per row from kAttnRowsMin (64) rows, where the per-row
// kernel's 148 persistent CTAs outrun the split-key clusters looping over rows
// (and whenever the split-key kernel cannot take the call, e.g. more than 640
// keys per row); the split-key cluster kernel below that; the general kernel
// for other shapes.
int launch_attn(const AttnArgs &a, cudaStream_t s) {
    const int64_t rows = (int64_t)a.B * a.Nq;
    const bool rows_ok = attn_rows_supported(a);
    if (rows_ok && (rows >= kAttnRowsMin || !attn_tc_supported(a))) return launch_attn_rows(a, s);
    if (attn_tc_supported(a)) return launch_attn_tc(a, s);
    return launch_attn_general(a, s);
}

}  // namespace csa2
