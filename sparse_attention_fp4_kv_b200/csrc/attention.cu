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
// General kernel (shapes outside the tensor-core kernels' constraints: other
// channel and head counts, e.g. 8 heads of 128 channels). The keys of a query
// are split over a cluster of NS CTAs (up to 8); each CTA serves a group of 8
// heads, so every key row is read once per head group, and the CTAs exchange
// their partial softmax results through distributed shared memory.
//  1. The CTA's keys, in chunks that fit in shared memory: positions, then
//     every row dequantized into a bf16 tile (E2M1 x E4M3 or x E8M0 has at
//     most 6 significant bits, so bf16 holds it exactly; window rows are bf16).
//  2. Logits: warp w takes keys w, w + 8, ...; lane l holds channel pairs
//     l, l + 32, ... of the 8 heads' Q; the 8 dot products are reduced across
//     the warp by a transposing butterfly (9 shuffles), lane 4h + i ends with
//     head h's logit.
//  3. Online softmax and P V: warp h owns head h, rescales its running output
//     (the lane's channels, in registers) and accumulates p_j row_j.
//  4. Combine: each CTA publishes (m, l, O) in shared memory; after a cluster
//     barrier, CTA r combines the heads h with h % NS == r from all NS CTAs.
// Every loop stays rolled: a call runs once per layer on an instruction cache
// that the kernels before it have emptied.
#include "attention.cuh"

namespace csa2 {

constexpr int GEN_THREADS = 256;
constexpr int GEN_WARPS = GEN_THREADS / 32;
constexpr int GEN_HG = 8;                  // heads per CTA: one warp per head in steps 3-4
constexpr int GEN_MAX_NS = 8;              // CTAs per cluster (portable cluster size)
constexpr size_t GEN_TILE_BYTES = 96 * 1024;  // bf16 key tile per chunk
// Dynamic shared memory the kernel is set up for: the tile plus Q/O (8 x 1024
// fp32) and the logits and positions of the chunk (at most 41 KB more).
constexpr size_t GEN_SMEM_LIMIT = 160 * 1024;
static_assert(GEN_HG == GEN_WARPS, "one warp per head");

struct GenGeom {
    int ns;   // CTAs per cluster (key splits)
    int kpc;  // keys per CTA (the last CTA of a query may hold fewer)
    int kch;  // keys per chunk
};

__device__ __forceinline__ uint32_t gen_cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void gen_cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
// Address of this CTA's shared variable p in the shared memory of cluster CTA r.
__device__ __forceinline__ uint32_t gen_dsmem(const void *p, uint32_t r) {
    uint32_t a = (uint32_t)__cvta_generic_to_shared(p), out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(a), "r"(r));
    return out;
}
__device__ __forceinline__ float gen_ld_remote(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ float2 gen_ld_remote2(uint32_t addr) {
    float2 v;
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr)
                 : "memory");
    return v;
}

// Dequantizes 32 channels (16 code bytes, two scales) into 16 bf16 pairs.
__device__ __forceinline__ void gen_dequant32(uint2 lo, uint2 hi, float s0, float s1, uint4 *dst) {
    const uint32_t w[4] = {lo.x, lo.y, hi.x, hi.y};
#pragma unroll
    for (int q = 0; q < 4; q++) {
        const float sc = q < 2 ? s0 : s1;
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const uint32_t byte = (w[q] >> (8 * e)) & 0xFFu;
            const float x = e2m1_to_f32(byte & 0xFu) * sc, y = e2m1_to_f32(byte >> 4) * sc;
            o[e] = (__float_as_uint(x) >> 16) | (__float_as_uint(y) & 0xFFFF0000u);  // exact
        }
        dst[q] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

template <int NPL>  // channel pairs per lane (C / 64, rounded up to a power of two)
__global__ void __launch_bounds__(GEN_THREADS) attn_general_kernel(AttnArgs a, GenGeom g) {
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ __align__(16) uint8_t gsm[];
    const int C = a.C, npairs = C / 2, nch = C / 32;
    uint32_t *tile = reinterpret_cast<uint32_t *>(gsm);                           // [kch][C/2] bf16x2
    float *qo = reinterpret_cast<float *>(gsm + (size_t)g.kch * C * 2);          // [8][C] Q, then O
    float *lg = qo + GEN_HG * C;                                                   // [8][kch]
    int32_t *kpos = reinterpret_cast<int32_t *>(lg + GEN_HG * g.kch);             // [kch]
    __shared__ float m_sh[GEN_HG], l_sh[GEN_HG];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = gen_cluster_rank();
    const int h0 = blockIdx.y * GEN_HG;
    const int64_t rows = (int64_t)a.B * a.Nq;
    for (int64_t bq = blockIdx.z; bq < rows; bq += gridDim.z) {
        const int b = (int)(bq / a.Nq);
        const AttnWindow w = attn_window(a, b, bq);
        const int nkeys = a.K + w.n;
        const int j_beg = (int)rank * g.kpc;
        const int j_end = min(nkeys, j_beg + g.kpc);
        // positions of the first chunk (see 1a), loaded together with Q
        const int kn0 = max(0, min(g.kch, j_end - j_beg));
        int32_t pos0 = -1;
        if (tid < kn0) {
            const int jj = j_beg + tid;
            if (jj < a.K) {
                const int32_t pos = a.topk[bq * a.K + jj];
                pos0 = (pos >= 0 && pos < a.cap) ? pos : -1;
            } else {
                pos0 = -2 - (int32_t)(w.row0 + (jj - a.K));
            }
        }
        // Q of the 8 heads as fp32 (heads beyond Hq read as zero)
#pragma unroll 4
        for (int i = tid; i < GEN_HG * npairs; i += GEN_THREADS) {
            const int h = i / npairs, p = i - h * npairs;
            uint32_t u = 0;
            if (h0 + h < a.Hq)
                u = __ldg(reinterpret_cast<const uint32_t *>(a.q) + (bq * a.Hq + h0 + h) * (int64_t)npairs + p);
            qo[h * C + 2 * p] = bf16_lo(u);
            qo[h * C + 2 * p + 1] = bf16_hi(u);
        }
        // running softmax state of head `warp` (warp-uniform) and its output
        float m_run = -INFINITY, l_run = 0.0f;
        float2 acc[NPL];
#pragma unroll
        for (int i = 0; i < NPL; i++) acc[i] = make_float2(0.0f, 0.0f);
        for (int c0 = j_beg; c0 < j_end; c0 += g.kch) {
            const int kn = min(g.kch, j_end - c0);
            __syncthreads();  // the previous chunk's tile and logits are consumed
            // 1a. positions (-1: empty slot; window rows as -2 - row); the first
            // chunk's first GEN_THREADS came with Q
            if (c0 == j_beg && tid < kn) kpos[tid] = pos0;
            for (int j = (c0 == j_beg ? tid + GEN_THREADS : tid); j < kn; j += GEN_THREADS) {
                const int jj = c0 + j;
                int32_t v;
                if (jj < a.K) {
                    const int32_t pos = a.topk[bq * a.K + jj];
                    v = (pos >= 0 && pos < a.cap) ? pos : -1;
                } else {
                    v = -2 - (int32_t)(w.row0 + (jj - a.K));
                }
                kpos[j] = v;
            }
            __syncthreads();
            // 1b. rows into the tile, 32 channels per item: the chunk's
            // selected rows [0, nf), then its window rows [nf, kn)
            const int nf = max(0, min(kn, a.K - c0));
#pragma unroll 2
            for (int it = tid; it < nf * nch; it += GEN_THREADS) {
                const int j = it / nch, c32 = it - j * nch;
                const int32_t v = kpos[j];
                if (v < 0) {  // empty slot: logit -inf, a zero row (p = 0 times it stays 0)
                    uint4 *dst = reinterpret_cast<uint4 *>(tile + (size_t)j * npairs + 16 * c32);
#pragma unroll
                    for (int q = 0; q < 4; q++) dst[q] = make_uint4(0, 0, 0, 0);
                    continue;
                }
                const int64_t cell = (int64_t)b * a.cap + v;
                const uint8_t *row = a.kv_fp4 + cell * (C / 2) + 16 * c32;
                const uint2 lo = __ldg(reinterpret_cast<const uint2 *>(row));
                const uint2 hi = __ldg(reinterpret_cast<const uint2 *>(row + 8));
                float s0, s1;
                if (a.mx) {
                    s0 = s1 = e8m0_to_f32(__ldg(a.kv_sf + cell * (C / 32) + c32));
                } else {
                    const uint8_t *sf = a.kv_sf + cell * (C / 16) + 2 * c32;
                    s0 = e4m3_to_f32(__ldg(sf));
                    s1 = e4m3_to_f32(__ldg(sf + 1));
                }
                gen_dequant32(lo, hi, s0, s1, reinterpret_cast<uint4 *>(tile + (size_t)j * npairs + 16 * c32));
            }
#pragma unroll 2
            for (int it = nf * nch + tid; it < kn * nch; it += GEN_THREADS) {
                const int j = it / nch, c32 = it - j * nch;
                const int64_t wrow = -2 - kpos[j];
                const uint4 *src = reinterpret_cast<const uint4 *>(a.swa) +
                                   (((int64_t)b * a.swa_rows + wrow) * C * 2 + 64 * c32) / 16;
                uint4 *dst = reinterpret_cast<uint4 *>(tile + (size_t)j * npairs + 16 * c32);
#pragma unroll
                for (int q = 0; q < 4; q++) dst[q] = __ldg(src + q);
            }
            __syncthreads();
            // 2. logits of the 8 heads
            // with at most 2 channel pairs per lane the 8 heads' Q stay in registers
            constexpr int QR = NPL <= 2 ? NPL : 1;
            float2 qr[GEN_HG][QR];
#pragma unroll
            for (int h = 0; h < GEN_HG; h++)
#pragma unroll
                for (int i = 0; i < QR; i++) {
                    const int p = lane + 32 * i;
                    qr[h][i] = (NPL <= 2 && p < npairs) ? *reinterpret_cast<const float2 *>(qo + h * C + 2 * p)
                                                        : make_float2(0.0f, 0.0f);
                }
#pragma unroll 1
            for (int j = warp; j < kn; j += GEN_WARPS) {
                float d[GEN_HG];
#pragma unroll
                for (int h = 0; h < GEN_HG; h++) d[h] = 0.0f;
#pragma unroll
                for (int i = 0; i < NPL; i++) {
                    const int p = lane + 32 * i;
                    if (p < npairs) {
                        const uint32_t kw = tile[(size_t)j * npairs + p];
                        const float kx = bf16_lo(kw), ky = bf16_hi(kw);
#pragma unroll
                        for (int h = 0; h < GEN_HG; h++) {
                            const float2 qq = NPL <= 2 ? qr[h][i < QR ? i : 0]
                                                       : *reinterpret_cast<const float2 *>(qo + h * C + 2 * p);
                            d[h] = fmaf(qq.x, kx, fmaf(qq.y, ky, d[h]));
                        }
                    }
                }
                // transposing butterfly: lanes with bit 4 keep heads 4-7, then
                // bit 3 halves again, bit 2 once more; bits 1 and 0 finish the sum
                const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
                float e4[4], e2[2];
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const float send = b4 ? d[i] : d[i + 4];
                    const float keep = b4 ? d[i + 4] : d[i];
                    e4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                }
#pragma unroll
                for (int i = 0; i < 2; i++) {
                    const float send = b3 ? e4[i] : e4[i + 2];
                    const float keep = b3 ? e4[i + 2] : e4[i];
                    e2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                }
                float e1 = (b2 ? e2[1] : e2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? e2[0] : e2[1], 4);
                e1 += __shfl_xor_sync(0xffffffffu, e1, 2);
                e1 += __shfl_xor_sync(0xffffffffu, e1, 1);
                if ((lane & 3) == 0) {
                    const int h = lane >> 2;  // = 4 b4 + 2 b3 + b2
                    lg[h * g.kch + j] = kpos[j] == -1 ? -INFINITY : e1 * a.scale;
                }
            }
            __syncthreads();
            // 3. online softmax and P V of head `warp`
            {
                float *lh = lg + warp * g.kch;
                float mc = -INFINITY;
                for (int j = lane; j < kn; j += 32) mc = fmaxf(mc, lh[j]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
                const float m_new = fmaxf(m_run, mc);
                if (m_new != -INFINITY) {
                    const float alpha = m_run == -INFINITY ? 0.0f : expf(m_run - m_new);
                    float z = 0.0f;
                    for (int j = lane; j < kn; j += 32) {
                        const float p = lh[j] == -INFINITY ? 0.0f : expf(lh[j] - m_new);
                        lh[j] = p;
                        z += p;
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
                    l_run = l_run * alpha + z;
                    m_run = m_new;
#pragma unroll
                    for (int i = 0; i < NPL; i++) {
                        acc[i].x *= alpha;
                        acc[i].y *= alpha;
                    }
                    __syncwarp();
                    // four keys per round, all their loads issued first (every row of
                    // the tile is finite: empty slots hold zeros)
#pragma unroll 1
                    for (int j0 = 0; j0 < kn; j0 += 4) {
                        float p[4];
                        uint32_t vw[4][NPL];
#pragma unroll
                        for (int u = 0; u < 4; u++) {
                            const int j = j0 + u;
                            p[u] = j < kn ? lh[j] : 0.0f;
#pragma unroll
                            for (int i = 0; i < NPL; i++) {
                                const int pp = lane + 32 * i;
                                vw[u][i] = (j < kn && pp < npairs) ? tile[(size_t)j * npairs + pp] : 0u;
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 4; u++)
#pragma unroll
                            for (int i = 0; i < NPL; i++) {
                                acc[i].x = fmaf(p[u], bf16_lo(vw[u][i]), acc[i].x);
                                acc[i].y = fmaf(p[u], bf16_hi(vw[u][i]), acc[i].y);
                            }
                    }
                }
            }
        }
        // 4. publish (m, l, O) of the 8 heads; Q is dead once every warp has
        // passed the last chunk's logits (or there was no chunk)
        __syncthreads();
#pragma unroll
        for (int i = 0; i < NPL; i++) {
            const int pp = lane + 32 * i;
            if (pp < npairs) *reinterpret_cast<float2 *>(qo + warp * C + 2 * pp) = acc[i];
        }
        if (lane == 0) {
            m_sh[warp] = m_run;
            l_sh[warp] = l_run;
        }
        gen_cluster_sync();
        const int h = warp;
        if (h % g.ns == (int)rank && h0 + h < a.Hq) {
            // every source's statistics with one round of remote loads
            float mr[GEN_MAX_NS], lr[GEN_MAX_NS];
#pragma unroll
            for (int r = 0; r < GEN_MAX_NS; r++) {
                mr[r] = r < g.ns ? gen_ld_remote(gen_dsmem(&m_sh[h], r)) : -INFINITY;
                lr[r] = r < g.ns ? gen_ld_remote(gen_dsmem(&l_sh[h], r)) : 0.0f;
            }
            float m_all = -INFINITY;
#pragma unroll
            for (int r = 0; r < GEN_MAX_NS; r++) m_all = fmaxf(m_all, mr[r]);
            float L = 0.0f;
            float2 o[NPL];
#pragma unroll
            for (int i = 0; i < NPL; i++) o[i] = make_float2(0.0f, 0.0f);
            if (m_all != -INFINITY) {
#pragma unroll
                for (int r = 0; r < GEN_MAX_NS; r++) {
                    if (r >= g.ns || mr[r] == -INFINITY) continue;
                    const float e = expf(mr[r] - m_all);
                    L += e * lr[r];
#pragma unroll
                    for (int i = 0; i < NPL; i++) {
                        const int pp = lane + 32 * i;
                        if (pp < npairs) {
                            const float2 v = gen_ld_remote2(gen_dsmem(qo + h * C + 2 * pp, r));
                            o[i].x = fmaf(e, v.x, o[i].x);
                            o[i].y = fmaf(e, v.y, o[i].y);
                        }
                    }
                }
            }
            const float inv = L > 0.0f ? 1.0f / L : 0.0f;
            float *out = a.out + (bq * a.Hq + h0 + h) * (int64_t)C;
#pragma unroll
            for (int i = 0; i < NPL; i++) {
                const int pp = lane + 32 * i;
                if (pp < npairs)
                    *reinterpret_cast<float2 *>(out + 2 * pp) = make_float2(o[i].x * inv, o[i].y * inv);
            }
        }
        gen_cluster_sync();  // no CTA reuses or leaves its shared memory while others read it
    }
}

static GenGeom gen_geometry(const AttnArgs &a) {
    const int win = a.swa_rows > 0 && a.swa && a.n_win > 0 ? (a.n_win < a.swa_rows ? a.n_win : a.swa_rows) : 0;
    const int T = a.K + win;  // most keys of one query
    GenGeom g;
    g.ns = (T + 63) / 64;  // about 64 keys or more per CTA
    if (g.ns < 1) g.ns = 1;
    if (g.ns > GEN_MAX_NS) g.ns = GEN_MAX_NS;
    g.kpc = T > 0 ? (T + g.ns - 1) / g.ns : 1;
    const int fit = (int)(GEN_TILE_BYTES / ((size_t)a.C * 2));
    g.kch = g.kpc < fit ? g.kpc : fit;
    return g;
}

static size_t gen_smem_bytes(const AttnArgs &a, const GenGeom &g) {
    return (size_t)g.kch * a.C * 2 + (size_t)GEN_HG * a.C * 4 + (size_t)GEN_HG * g.kch * 4 +
           (size_t)g.kch * 4;
}

template <int NPL>
static int launch_general(const AttnArgs &a, const GenGeom &g, size_t smem, cudaStream_t s) {
    static PerDevice smem_set;
    if (!set_smem_limit_once(smem_set, attn_general_kernel<NPL>, GEN_SMEM_LIMIT)) return CSA2_ERR_CUDA;
    const int64_t rows = (int64_t)a.B * a.Nq;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)g.ns, (unsigned)((a.Hq + GEN_HG - 1) / GEN_HG),
                       (unsigned)(rows < 65535 ? rows : 65535));
    cfg.blockDim = dim3(GEN_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)g.ns;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, attn_general_kernel<NPL>, a, g) != cudaSuccess) return CSA2_ERR_CUDA;
    return launch_status();
}

int launch_attn_general(const AttnArgs &a, cudaStream_t s) {
    const GenGeom g = gen_geometry(a);
    const size_t smem = gen_smem_bytes(a, g);
    if (smem > GEN_SMEM_LIMIT) return CSA2_ERR_SHAPE;
    const int npl = (a.C / 2 + 31) / 32;  // 1 .. 16 (C <= 1024)
    if (npl <= 1) return launch_general<1>(a, g, smem, s);
    if (npl <= 2) return launch_general<2>(a, g, smem, s);
    if (npl <= 4) return launch_general<4>(a, g, smem, s);
    if (npl <= 8) return launch_general<8>(a, g, smem, s);
    return launch_general<16>(a, g, smem, s);
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
    if (!aligned(a.ws, 16)) return CSA2_ERR_ALIGN;  // 16-byte accesses to the exchange slots
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
