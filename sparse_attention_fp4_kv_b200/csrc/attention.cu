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
// General kernel: one CTA per (query, head), 16 warps when a lane holds at
// most 2 channel pairs (C <= 128), else 8. Lane l of a warp holds
// channel pairs l, l + 32, ... (pair i = channels 2i, 2i + 1 = one FP4 byte).
//  1. The query's selected positions go to shared memory.
//  2. Logits: warp w takes keys in runs of U (= 32 / NP, at least 2: as many
//     as the registers hold) with all their loads issued before the first use;
//     fp32 dot, shuffle reduce.
//  3. Softmax statistics over the logits in shared memory.
//  4. P V: warp w accumulates p_j row_j over the same keys in registers (the
//     lane's channels), U keys per round; the warps' sums are added in shared
//     memory.
// Used for shapes outside the tensor-core kernels' constraints (other channel
// and head counts, e.g. 8 heads of 128 channels).
#include "attention.cuh"

namespace csa2 {

// threads of the CTA for NP channel pairs per lane
template <int NP>
constexpr int gen_threads() { return NP <= 2 ? 512 : 256; }
constexpr int GEN_MAX_WARPS = 16;
// keys per warp per round with NP channel pairs per lane
template <int NP>
constexpr int gen_keys_per_round() { return NP >= 16 ? 2 : 32 / NP; }

// Key j of query bq (j < K: selected row, else window row j - K) as NP channel
// pairs per lane, dequantized; valid = false for an empty selected slot.
template <int NP>
__device__ __forceinline__ void gen_load_key(const AttnArgs &a, int b, const int32_t *sel,
                                             const AttnWindow &w, int j, int lane, float2 (&v)[NP],
                                             bool &valid) {
    const int C = a.C, npairs = C / 2;
    if (j < a.K) {
        const int32_t pos = sel[j];
        valid = pos >= 0 && pos < a.cap;
        const int64_t cell = (int64_t)b * a.cap + (valid ? pos : 0);
        const uint8_t *row = a.kv_fp4 + cell * (C / 2);
        const uint8_t *sfr = a.kv_sf + cell * (C / (a.mx ? 32 : 16));
        uint32_t byte[NP];
        float sc[NP];
#pragma unroll
        for (int i = 0; i < NP; i++) {
            const int p = lane + 32 * i;
            byte[i] = p < npairs ? __ldg(row + p) : 0u;
            sc[i] = p < npairs ? kv_group_scale(sfr, p >> 3, a.mx) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < NP; i++)
            v[i] = valid ? make_float2(e2m1_to_f32(byte[i] & 0xF) * sc[i], e2m1_to_f32(byte[i] >> 4) * sc[i])
                         : make_float2(0.0f, 0.0f);
    } else {
        valid = true;
        const uint32_t *row = reinterpret_cast<const uint32_t *>(a.swa) +
                              ((int64_t)b * a.swa_rows + w.row0 + (j - a.K)) * (C / 2);
#pragma unroll
        for (int i = 0; i < NP; i++) {
            const int p = lane + 32 * i;
            const uint32_t u = p < npairs ? __ldg(row + p) : 0u;
            v[i] = make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
        }
    }
}

template <int NP>
__global__ void __launch_bounds__(gen_threads<NP>()) attn_general_kernel(AttnArgs a) {
    constexpr int GEN_U = gen_keys_per_round<NP>();
    constexpr int GEN_THREADS = gen_threads<NP>();
    constexpr int GEN_WARPS = GEN_THREADS / 32;
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ float sm[];
    const int C = a.C, npairs = C / 2;
    float *lg = sm;                                    // [K + n_win] logits, then p
    float *red = sm + a.K + a.n_win;                   // [warps][C] partial sums
    int32_t *sel = reinterpret_cast<int32_t *>(red + GEN_WARPS * C);  // [K]
    __shared__ float wred[GEN_MAX_WARPS];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bq = blockIdx.x / a.Hq;
    const int h = (int)(blockIdx.x % a.Hq);
    const int b = (int)(bq / a.Nq);
    const AttnWindow w = attn_window(a, b, bq);
    const int nkeys = a.K + w.n;
    for (int j = tid; j < a.K; j += GEN_THREADS) sel[j] = a.topk[bq * a.K + j];

    // this lane's query channels
    const uint32_t *q = reinterpret_cast<const uint32_t *>(a.q) + (bq * a.Hq + h) * (int64_t)(C / 2);
    float2 qv[NP];
#pragma unroll
    for (int i = 0; i < NP; i++) {
        const int p = lane + 32 * i;
        const uint32_t u = p < npairs ? __ldg(q + p) : 0u;
        qv[i] = make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
    __syncthreads();

    // ---- logits
    for (int j0 = warp * GEN_U; j0 < nkeys; j0 += GEN_WARPS * GEN_U) {
        float2 v[GEN_U][NP];
        bool valid[GEN_U];
#pragma unroll
        for (int u = 0; u < GEN_U; u++) {
            valid[u] = false;
            if (j0 + u < nkeys) gen_load_key<NP>(a, b, sel, w, j0 + u, lane, v[u], valid[u]);
        }
#pragma unroll
        for (int u = 0; u < GEN_U; u++) {
            float dot = 0.0f;
#pragma unroll
            for (int i = 0; i < NP; i++) dot += qv[i].x * v[u][i].x + qv[i].y * v[u][i].y;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            if (lane == 0 && j0 + u < nkeys) lg[j0 + u] = valid[u] ? dot * a.scale : -INFINITY;
        }
    }
    __syncthreads();

    // ---- softmax statistics
    float m = -INFINITY;
    for (int j = tid; j < nkeys; j += GEN_THREADS) m = fmaxf(m, lg[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wred[warp] = m;
    __syncthreads();
    m = -INFINITY;
    for (int w2 = 0; w2 < GEN_WARPS; w2++) m = fmaxf(m, wred[w2]);
    __syncthreads();
    float z = 0.0f;
    for (int j = tid; j < nkeys; j += GEN_THREADS) {
        const float p = (lg[j] == -INFINITY) ? 0.0f : expf(lg[j] - m);
        lg[j] = p;
        z += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane == 0) wred[warp] = z;
    __syncthreads();
    z = 0.0f;
    for (int w2 = 0; w2 < GEN_WARPS; w2++) z += wred[w2];
    const float inv = z > 0.0f ? 1.0f / z : 0.0f;

    // ---- P V over the same keys
    float2 acc[NP];
#pragma unroll
    for (int i = 0; i < NP; i++) acc[i] = make_float2(0.0f, 0.0f);
    for (int j0 = warp * GEN_U; j0 < nkeys; j0 += GEN_WARPS * GEN_U) {
        float2 v[GEN_U][NP];
        bool valid[GEN_U];
#pragma unroll
        for (int u = 0; u < GEN_U; u++) {
            valid[u] = false;
            if (j0 + u < nkeys && lg[j0 + u] != 0.0f) gen_load_key<NP>(a, b, sel, w, j0 + u, lane, v[u], valid[u]);
        }
#pragma unroll
        for (int u = 0; u < GEN_U; u++) {
            if (!valid[u]) continue;
            const float p = lg[j0 + u];
#pragma unroll
            for (int i = 0; i < NP; i++) {
                acc[i].x += p * v[u][i].x;
                acc[i].y += p * v[u][i].y;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NP; i++) {
        const int p = lane + 32 * i;
        if (p < npairs) {
            red[warp * C + 2 * p] = acc[i].x;
            red[warp * C + 2 * p + 1] = acc[i].y;
        }
    }
    __syncthreads();
    float *out = a.out + (bq * a.Hq + h) * (int64_t)C;
    for (int c = tid; c < C; c += GEN_THREADS) {
        float sum = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < GEN_WARPS; w2++) sum += red[w2 * C + c];
        out[c] = sum * inv;
    }
}

template <int NP>
static int launch_general(const AttnArgs &a, size_t smem, int64_t grid, cudaStream_t s) {
    static PerDevice smem_set;
    if (smem > 48 * 1024 && !set_smem_limit_once(smem_set, attn_general_kernel<NP>, 227 * 1024))
        return CSA2_ERR_CUDA;
    return launch_kernel(a.pdl, attn_general_kernel<NP>, dim3((unsigned)grid), dim3(gen_threads<NP>()),
                         smem, s, a);
}

int launch_attn_general(const AttnArgs &a, cudaStream_t s) {
    // logits [K + n_win], partial sums [warps][C], selected positions [K]
    const int pairs_per_lane = (a.C / 2 + 31) / 32;  // 1 .. 16 (C <= 1024)
    const int warps = pairs_per_lane <= 2 ? 16 : 8;
    const size_t smem = sizeof(float) * ((size_t)a.K + a.n_win + (size_t)warps * a.C) +
                        sizeof(int32_t) * (size_t)a.K;
    if (smem > 227 * 1024) return CSA2_ERR_SHAPE;
    const int64_t grid = (int64_t)a.B * a.Nq * a.Hq;
    if (grid > INT32_MAX) return CSA2_ERR_SHAPE;
    if (pairs_per_lane <= 1) return launch_general<1>(a, smem, grid, s);
    if (pairs_per_lane <= 2) return launch_general<2>(a, smem, grid, s);
    if (pairs_per_lane <= 4) return launch_general<4>(a, smem, grid, s);
    if (pairs_per_lane <= 8) return launch_general<8>(a, smem, grid, s);
    return launch_general<16>(a, smem, grid, s);
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
    return attn_call(a, ws_bytes, (cudaStream_t)stream);
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
    return attn_call(a, ws_bytes, (cudaStream_t)stream);
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
    if ((a.ws == nullptr ? 0 : ws_bytes) < attn_scratch_bytes(a.B, a.Nq, a.Hq, a.C, a.K))
        return CSA2_ERR_WORKSPACE;
    if ((int64_t)a.B * a.Nq == 0 || validate_only) return CSA2_OK;
    return launch_attn(a, s);
}

// A standalone call: its workspace starts with the call's error word, cleared
// at the call's start; the kernels' scratch follows it.
int attn_call(AttnArgs a, size_t ws_bytes, cudaStream_t s) {
    const size_t need = attn_workspace_bytes(a.B, a.Nq, a.Hq, a.C, a.K, a.n_win);
    if (need == 0) return attn_checked_launch(a, ws_bytes, s);
    if (a.ws == nullptr || ws_bytes < need) return CSA2_ERR_WORKSPACE;
    a.err = static_cast<int *>(a.ws);
    if (cudaMemsetAsync(a.err, 0, sizeof(int), s) != cudaSuccess) return CSA2_ERR_CUDA;
    a.ws = static_cast<char *>(a.ws) + kErrWordBytes;
    return attn_checked_launch(a, ws_bytes - kErrWordBytes, s);
}

// Scratch of the kernels (a.ws): the cluster kernel's exchange slots for its
// per-CTA partial results when its shape constraints could hold; the other
// kernels need none.
size_t attn_scratch_bytes(int B, int Nq, int Hq, int C, int K) {
    if (C == 512 && Hq == 64 && K > 0 && K <= 640) return attn_tc_workspace_bytes(B, Nq);
    return 0;
}

// Workspace of a standalone call: the call's error word (kErrWordBytes)
// whenever a tensor-core kernel, whose waits are bounded, may take the call
// (512 channels, 64 heads), followed by the kernels' scratch. The general
// kernel waits on nothing and needs none.
size_t attn_workspace_bytes(int B, int Nq, int Hq, int C, int K, int n_win) {
    (void)n_win;
    if (C != 512 || Hq != 64) return 0;
    return kErrWordBytes + attn_scratch_bytes(B, Nq, Hq, C, K);
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
