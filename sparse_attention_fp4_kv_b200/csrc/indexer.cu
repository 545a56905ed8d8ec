// Indexer kernels: Full-layer scan (token scores + 8-token block maxima),
// Reindex rescoring of the pooled blocks, and the pool gather of the Full
// layer's own token scores.
//
// "DeepSeek-V4.1-Flash: 890 Bytes Per Token, 437x Smaller KV Cache", CSA2
// section: a Full layer scores the context with its indexer and builds the
// pool of up to 2,048 blocks of 8 tokens; a Reindex layer rescores that pool
// with its own indexer Q. "DeepSeek V4.1 Flash KV Cache: 890 Bytes per Token
// Explained", indexer section: deeper layers search only the pool, so indexer
// work grows with the pool, not with the context.
//
// Score of token t for query q: S = sum over heads and dims of q*k (int8 x
// int8, int32 accumulate with dp4a), score = fp32_rn(S) * k_scale[t].
//
// Decode has one query per sequence, so the scan is a pure stream over the
// indexer keys (2 KB per token at 16 x 128): HBM bound, with no operand reuse
// for tensor cores. One warp scores one 8-token block (16 KB contiguous at
// 16 x 128): every lane issues 16-byte streaming loads (L1 no-allocate, L2
// evict-first), the int32 partial sums of the 8 tokens are combined by a
// 9-shuffle transpose-reduce, and the block maximum by 3 more. A persistent
// grid of warps walks the (query, block) items with a stride of the total warp
// count, so neighbouring warps read neighbouring blocks.
#include <cfloat>

#include "common.cuh"

namespace csa2 {

// Lane -> token of the 8-token block whose full sum the lane holds after the
// transpose-reduce (bits 4, 3, 2 of the lane id).
__device__ __forceinline__ int reduce_token_of_lane(int lane) {
    return ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
}

// Warp-wide: part[t] (lane partial sums of token t) -> full sum of token
// reduce_token_of_lane(lane).
__device__ __forceinline__ int transpose_reduce8(const int (&part)[8], int lane) {
    int q4[4], q2[2];
    const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4;
#pragma unroll
    for (int t = 0; t < 4; t++) {
        int send = u16 ? part[t] : part[t + 4];
        int keep = u16 ? part[t + 4] : part[t];
        q4[t] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int t = 0; t < 2; t++) {
        int send = u8 ? q4[t] : q4[t + 2];
        int keep = u8 ? q4[t + 2] : q4[t];
        q2[t] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    int send = u4 ? q2[0] : q2[1];
    int keep = u4 ? q2[1] : q2[0];
    int s = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    return s;
}

__device__ __forceinline__ int dot16(const uint4 &k, const uint4 &q, int acc) {
    acc = __dp4a((int)k.x, (int)q.x, acc);
    acc = __dp4a((int)k.y, (int)q.y, acc);
    acc = __dp4a((int)k.z, (int)q.z, acc);
    acc = __dp4a((int)k.w, (int)q.w, acc);
    return acc;
}

// Rows of HD bytes, split into VPT 16-byte vectors. An 8-token block is
// 8 * VPT vectors; lane l takes vectors 32 * i + l.
template <int HD>
struct RowShape {
    static_assert(HD % 16 == 0, "row must be a whole number of 16-byte vectors");
    static constexpr int VPT = HD / 16;
    static constexpr int VPL = (8 * VPT + 31) / 32;  // vectors per lane per block
    static constexpr int QV = VPT >= 32 ? VPT / 32 : 1;
    static_assert(VPT >= 32 ? VPT % 32 == 0 : 32 % VPT == 0, "unsupported row size");
};

template <int HD>
__device__ __forceinline__ void load_qfrag(const int8_t *q, uint4 (&qf)[RowShape<HD>::QV], int lane) {
    using RS = RowShape<HD>;
    const uint4 *qv = reinterpret_cast<const uint4 *>(q);
#pragma unroll
    for (int j = 0; j < RS::QV; j++) qf[j] = qv[RS::VPT >= 32 ? 32 * j + lane : lane % RS::VPT];
}

// Exact int32 dot products of the block's ntok (1..8) tokens with the query;
// returns the sum for token reduce_token_of_lane(lane) (0 for t >= ntok).
// GROUP = 16-byte loads each lane has in flight before it uses them.
template <int HD, int GROUP = 8>
__device__ __forceinline__ int block_dots(const int8_t *kblk, const uint4 (&qf)[RowShape<HD>::QV],
                                          int lane, int ntok) {
    using RS = RowShape<HD>;
    const uint4 *kv = reinterpret_cast<const uint4 *>(kblk);
    int part[8];
#pragma unroll
    for (int t = 0; t < 8; t++) part[t] = 0;
#pragma unroll
    for (int i0 = 0; i0 < RS::VPL; i0 += GROUP) {
        uint4 k[GROUP];
#pragma unroll
        for (int u = 0; u < GROUP; u++) {
            const int i = i0 + u;
            if (i < RS::VPL) {
                const int v = 32 * i + lane;
                const int tok = v / RS::VPT;
                k[u] = (tok < ntok) ? ld_stream_v4(kv + v) : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < GROUP; u++) {
            const int i = i0 + u;
            if (i < RS::VPL) {
                const int v = 32 * i + lane;
                const int tok = v / RS::VPT;
                const int s = dot16(k[u], qf[RS::VPT >= 32 ? i % RS::QV : 0], 0);
#pragma unroll
                for (int t = 0; t < 8; t++) part[t] += (tok == t) ? s : 0;
            }
        }
    }
    return transpose_reduce8(part, lane);
}

// Generic-row variant (any HD % 16 == 0): the warp walks the block token by
// token; lanes stride over the row's vectors. Returns the full sum of token
// reduce_token_of_lane(lane), matching block_dots.
__device__ __forceinline__ int block_dots_generic(const int8_t *kblk, const int8_t *q, int HD,
                                                  int lane, int ntok) {
    const int VPT = HD / 16;
    const uint4 *kv = reinterpret_cast<const uint4 *>(kblk);
    const uint4 *qv = reinterpret_cast<const uint4 *>(q);
    const int my_tok = reduce_token_of_lane(lane);
    int mine = 0;
    for (int t = 0; t < ntok; t++) {
        int s = 0;
        for (int c = lane; c < VPT; c += 32) s = dot16(ld_stream_v4(kv + (int64_t)t * VPT + c), qv[c], s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (t == my_tok) mine = s;
    }
    return mine;
}

// Score of the lane's token (or -inf if it is not visible) and the block max.
__device__ __forceinline__ float lane_score(int S, const float *kscale_blk, int tok, int ntok) {
    return tok < ntok ? __fmul_rn(__int2float_rn(S), kscale_blk[tok]) : -FLT_MAX * 2.0f;
}

__device__ __forceinline__ float warp_block_max(float s) {
    s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 4));
    s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 8));
    s = fmaxf(s, __shfl_xor_sync(0xffffffffu, s, 16));
    return s;
}

// ------------------------------------------------------------------ Full scan
struct ScanArgs {
    const int8_t *q;
    const int8_t *k;
    const float *kscale;
    const int64_t *ctx_len;
    const int64_t *q_pos;
    int B, Nq, HD;
    int64_t cap, nblk_cap;
    float *tok;
    float *blk;
    int32_t *n_blk;
    uint32_t *hist;  // optional [B*Nq][4096] counts of block scores by first digit
};

template <int HD>
__global__ void __launch_bounds__(256) index_full_kernel(ScanArgs a) {
    grid_dep_wait();
    grid_dep_launch();
    using RS = RowShape<HD>;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t items = (int64_t)a.B * a.Nq * a.nblk_cap;
    const int my_tok = reduce_token_of_lane(lane);
    int64_t cur_bq = -1;
    int64_t V = 0;
    uint4 qf[RS::QV];
    for (int64_t it = warp; it < items; it += nwarps) {
        const int64_t bq = it / a.nblk_cap;
        const int64_t j = it - bq * a.nblk_cap;
        const int b = (int)(bq / a.Nq), i = (int)(bq % a.Nq);
        if (bq != cur_bq) {
            cur_bq = bq;
            V = visible_len(a.ctx_len, a.q_pos, b, i, a.Nq);
            if (V > a.cap) V = a.cap;
            load_qfrag<HD>(a.q + bq * HD, qf, lane);
        }
        if (j == 0 && lane == 0 && a.n_blk) a.n_blk[bq] = (int32_t)((V + 7) / 8);
        if (8 * j >= V) continue;
        const int ntok = (int)(V - 8 * j < 8 ? V - 8 * j : 8);
        const int64_t t0 = (int64_t)b * a.cap + 8 * j;
        const int S = block_dots<HD>(a.k + t0 * HD, qf, lane, ntok);
        const float sc = lane_score(S, a.kscale + t0, my_tok, ntok);
        const float m = warp_block_max(sc);
        if (a.tok && (lane & 3) == 0 && my_tok < ntok) a.tok[bq * a.cap + 8 * j + my_tok] = sc;
        if (lane == 0) {
            a.blk[bq * a.nblk_cap + j] = m;
            if (a.hist) atomicAdd(&a.hist[bq * kHistBins + hist_bin(m)], 1u);
        }
    }
}

__global__ void __launch_bounds__(256) index_full_generic_kernel(ScanArgs a) {
    grid_dep_wait();
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t items = (int64_t)a.B * a.Nq * a.nblk_cap;
    const int my_tok = reduce_token_of_lane(lane);
    for (int64_t it = warp; it < items; it += nwarps) {
        const int64_t bq = it / a.nblk_cap;
        const int64_t j = it - bq * a.nblk_cap;
        const int b = (int)(bq / a.Nq), i = (int)(bq % a.Nq);
        int64_t V = visible_len(a.ctx_len, a.q_pos, b, i, a.Nq);
        if (V > a.cap) V = a.cap;
        if (j == 0 && lane == 0 && a.n_blk) a.n_blk[bq] = (int32_t)((V + 7) / 8);
        if (8 * j >= V) continue;
        const int ntok = (int)(V - 8 * j < 8 ? V - 8 * j : 8);
        const int64_t t0 = (int64_t)b * a.cap + 8 * j;
        const int S = block_dots_generic(a.k + t0 * a.HD, a.q + bq * a.HD, a.HD, lane, ntok);
        const float sc = lane_score(S, a.kscale + t0, my_tok, ntok);
        const float m = warp_block_max(sc);
        if (a.tok && (lane & 3) == 0 && my_tok < ntok) a.tok[bq * a.cap + 8 * j + my_tok] = sc;
        if (lane == 0) {
            a.blk[bq * a.nblk_cap + j] = m;
            if (a.hist) atomicAdd(&a.hist[bq * kHistBins + hist_bin(m)], 1u);
        }
    }
}

// ------------------------------------------------------------------ Reindex
struct ReindexArgs {
    const int8_t *q;
    const int8_t *k;
    const float *kscale;
    const int32_t *pool;
    const int64_t *ctx_len;
    const int64_t *q_pos;
    int B, Nq, HD, P;
    int64_t cap;
    float *pscore;
    int32_t *ppos;
    uint32_t *hist;  // optional [B*Nq][4096] counts of pooled scores by first digit
};

__device__ __forceinline__ int64_t reindex_block(const ReindexArgs &a, int64_t bq, int s, int64_t V,
                                                 int &ntok) {
    const int32_t blkid = a.pool[bq * a.P + s];
    ntok = 0;
    if (blkid < 0) return -1;
    const int64_t t0 = 8 * (int64_t)blkid;
    if (t0 >= V) return -1;
    ntok = (int)(V - t0 < 8 ? V - t0 : 8);
    return t0;
}

// A grid of warps walks the pooled blocks (items w, w + nwarps, ...; nwarps =
// the grid's warp count), 16 loads per lane in flight. Before its
// grid-dependency wait a warp finds its first block from the pool and the
// context lengths and pulls the block's keys into L2, so that with dependent
// launches the key stream overlaps the previous kernel (a latency-bound
// attention launch that leaves HBM idle). The pool comes from the Full layer's
// selection, which is always two or more kernels earlier (its attention
// follows it), and the keys and context lengths are not written during a
// step; the layer's own indexer query, the only input the previous kernel may
// produce, is read after the wait. The launch has one warp per block (the
// loop runs once): four blocks per warp, all prefetched, measured 1.725
// against 1.681 ms per 1M step (the prefetches overran L2), and a persistent
// grid of one resident wave 1.697 against 1.664 ms (same B200 each time).
// Four CTAs per SM (64 registers) instead of three take the grid from 2.3 to
// 1.7 waves: 1.635 to 1.624 ms per 1M step, 348 to 342 us per 32-row Reindex
// group step; five per SM would spill.
template <int HD>
__global__ void __launch_bounds__(256, 4) index_reindex_kernel(ReindexArgs a) {
    using RS = RowShape<HD>;
    const int lane = threadIdx.x & 31;
    const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t items = (int64_t)a.B * a.Nq * a.P;
    // item -> (query row, pool slot, sequence, first token (-1: empty), tokens)
    auto locate = [&](int64_t it, int64_t &bq, int &s, int &b, int64_t &t0, int &ntok) {
        bq = it / a.P;
        s = (int)(it - bq * a.P);
        b = (int)(bq / a.Nq);
        int64_t V = visible_len(a.ctx_len, a.q_pos, b, (int)(bq % a.Nq), a.Nq);
        if (V > a.cap) V = a.cap;
        t0 = reindex_block(a, bq, s, V, ntok);
    };
    int64_t bq = 0, t0 = -1;
    int s = 0, b = 0, ntok = 0;
    if (w0 < items) {
        locate(w0, bq, s, b, t0, ntok);
        if (t0 >= 0 && lane == 0)
            bulk_prefetch_l2(a.k + ((int64_t)b * a.cap + t0) * HD, (uint32_t)(ntok * HD));
    }
    grid_dep_wait();
    grid_dep_launch();
    const int my_tok = reduce_token_of_lane(lane);
    int64_t cur_bq = -1;
    uint4 qf[RS::QV];
    for (int64_t it = w0; it < items; it += nwarps) {
        if (it != w0) locate(it, bq, s, b, t0, ntok);
        const int64_t slot = bq * 8 * (int64_t)a.P + 8 * (int64_t)s;
        if (t0 < 0) {
            if (lane < 8) {
                a.ppos[slot + lane] = -1;
                a.pscore[slot + lane] = 0.0f;
            }
            continue;
        }
        if (bq != cur_bq) {
            cur_bq = bq;
            load_qfrag<HD>(a.q + bq * HD, qf, lane);
        }
        const int64_t row0 = (int64_t)b * a.cap + t0;
        const int S = block_dots<HD, 16>(a.k + row0 * HD, qf, lane, ntok);
        const float sc = lane_score(S, a.kscale + row0, my_tok, ntok);
        if ((lane & 3) == 0) {
            a.ppos[slot + my_tok] = my_tok < ntok ? (int32_t)(t0 + my_tok) : -1;
            a.pscore[slot + my_tok] = my_tok < ntok ? sc : 0.0f;
            if (a.hist && my_tok < ntok) atomicAdd(&a.hist[bq * kHistBins + hist_bin(sc)], 1u);
        }
    }
}

__global__ void __launch_bounds__(256) index_reindex_generic_kernel(ReindexArgs a) {
    grid_dep_wait();
    grid_dep_launch();
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t items = (int64_t)a.B * a.Nq * a.P;
    const int my_tok = reduce_token_of_lane(lane);
    for (int64_t it = warp; it < items; it += nwarps) {
        const int64_t bq = it / a.P;
        const int s = (int)(it - bq * a.P);
        const int b = (int)(bq / a.Nq), i = (int)(bq % a.Nq);
        int64_t V = visible_len(a.ctx_len, a.q_pos, b, i, a.Nq);
        if (V > a.cap) V = a.cap;
        int ntok;
        const int64_t t0 = reindex_block(a, bq, s, V, ntok);
        const int64_t slot = bq * 8 * (int64_t)a.P + 8 * (int64_t)s;
        if (t0 < 0) {
            if (lane < 8) {
                a.ppos[slot + lane] = -1;
                a.pscore[slot + lane] = 0.0f;
            }
            continue;
        }
        const int64_t row0 = (int64_t)b * a.cap + t0;
        const int S = block_dots_generic(a.k + row0 * a.HD, a.q + bq * a.HD, a.HD, lane, ntok);
        const float sc = lane_score(S, a.kscale + row0, my_tok, ntok);
        if ((lane & 3) == 0) {
            a.ppos[slot + my_tok] = my_tok < ntok ? (int32_t)(t0 + my_tok) : -1;
            a.pscore[slot + my_tok] = my_tok < ntok ? sc : 0.0f;
            if (a.hist && my_tok < ntok) atomicAdd(&a.hist[bq * kHistBins + hist_bin(sc)], 1u);
        }
    }
}

// ------------------------------------------------------------------ pool gather
__global__ void __launch_bounds__(256) pool_gather_kernel(const float *__restrict__ tok,
                                                          const int32_t *__restrict__ pool,
                                                          const int64_t *ctx_len,
                                                          const int64_t *q_pos, int B, int Nq,
                                                          int P, int64_t cap, float *pscore,
                                                          int32_t *ppos, uint32_t *hist) {
    grid_dep_wait();
    grid_dep_launch();
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = (int64_t)B * Nq * P * 8;
    if (idx >= total) return;
    const int r = (int)(idx & 7);
    const int64_t s_all = idx >> 3;
    const int64_t bq = s_all / P;
    const int b = (int)(bq / Nq), i = (int)(bq % Nq);
    int64_t V = visible_len(ctx_len, q_pos, b, i, Nq);
    if (V > cap) V = cap;
    const int32_t blkid = pool[s_all];
    const int64_t p = 8 * (int64_t)blkid + r;
    if (blkid >= 0 && p < V) {
        const float sc = tok[bq * cap + p];
        ppos[idx] = (int32_t)p;
        pscore[idx] = sc;
        if (hist) atomicAdd(&hist[bq * kHistBins + hist_bin(sc)], 1u);
    } else {
        ppos[idx] = -1;
        pscore[idx] = 0.0f;
    }
}

template <typename K>
static int persistent_grid(K kernel, int threads, int64_t items_warps) {
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, 0);
    if (occ <= 0) occ = 1;
    const int64_t want = (items_warps * 32 + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms() * occ;
    return (int)(want < cap ? (want < 1 ? 1 : want) : cap);
}

}  // namespace csa2

using namespace csa2;

static int dispatch_scan(const ScanArgs &a, cudaStream_t s, bool pdl) {
    const int64_t items = (int64_t)a.B * a.Nq * a.nblk_cap;
    const int T = 256;
    switch (a.HD) {
#define CSA2_SCAN_CASE(HDV)                                                             \
    case HDV: {                                                                         \
        int g = persistent_grid(index_full_kernel<HDV>, T, items);                      \
        return launch_kernel(pdl, index_full_kernel<HDV>, dim3(g), dim3(T), 0, s, a);  \
    }
        CSA2_SCAN_CASE(128)
        CSA2_SCAN_CASE(256)
        CSA2_SCAN_CASE(512)
        CSA2_SCAN_CASE(1024)
        CSA2_SCAN_CASE(2048)
        CSA2_SCAN_CASE(4096)
#undef CSA2_SCAN_CASE
        default: {
            int g = persistent_grid(index_full_generic_kernel, T, items);
            return launch_kernel(pdl, index_full_generic_kernel, dim3(g), dim3(T), 0, s, a);
        }
    }
}

static int dispatch_reindex(const ReindexArgs &a, cudaStream_t s, bool pdl) {
    const int64_t items = (int64_t)a.B * a.Nq * a.P;
    const int T = 256;
    switch (a.HD) {
#define CSA2_RI_CASE(HDV)                                                               \
    case HDV: {                                                                         \
        const int g = (int)((items + T / 32 - 1) / (T / 32));                            \
        return launch_kernel(pdl, index_reindex_kernel<HDV>, dim3((unsigned)g), dim3(T), 0, s, \
                             a);                                                        \
    }
        CSA2_RI_CASE(128)
        CSA2_RI_CASE(256)
        CSA2_RI_CASE(512)
        CSA2_RI_CASE(1024)
        CSA2_RI_CASE(2048)
        CSA2_RI_CASE(4096)
#undef CSA2_RI_CASE
        default: {
            int g = persistent_grid(index_reindex_generic_kernel, T, items);
            return launch_kernel(pdl, index_reindex_generic_kernel, dim3(g), dim3(T), 0, s, a);
        }
    }
}

static int check_indexer_common(const int8_t *q_idx, const int8_t *k_idx, const float *k_scale,
                                const int64_t *ctx_len, int B, int Nq, int H, int D, int64_t cap) {
    if (!q_idx || !k_idx || !k_scale || !ctx_len) return CSA2_ERR_NULL;
    if (B < 0 || Nq < 0 || H <= 0 || D <= 0 || cap < 1) return CSA2_ERR_SHAPE;
    const int64_t HD = (int64_t)H * D;
    if (HD % 16 || HD > 65536) return CSA2_ERR_SHAPE;
    if (!aligned(q_idx, 16) || !aligned(k_idx, 16)) return CSA2_ERR_ALIGN;
    return CSA2_OK;
}

extern "C" int csa2_index_full(const int8_t *q_idx, const int8_t *k_idx, const float *k_scale,
                               const int64_t *ctx_len, const int64_t *q_pos, int B, int Nq, int H,
                               int D, int64_t cap, float *tok_score, float *blk_score,
                               int32_t *n_blk, void *stream) {
    int st = check_indexer_common(q_idx, k_idx, k_scale, ctx_len, B, Nq, H, D, cap);
    if (st) return st;
    if (!blk_score) return CSA2_ERR_NULL;
    if ((int64_t)B * Nq == 0) return CSA2_OK;
    if (index_mma_supported(Nq, H * D, cap, B))
        return launch_index_mma(q_idx, k_idx, k_scale, ctx_len, q_pos, B, Nq, H * D, cap,
                                tok_score, blk_score, n_blk, (cudaStream_t)stream);
    ScanArgs a{q_idx, k_idx, k_scale, ctx_len, q_pos, B, Nq, H * D, cap, (cap + 7) / 8,
               tok_score, blk_score, n_blk, nullptr};
    return dispatch_scan(a, (cudaStream_t)stream, false);
}

extern "C" int csa2_index_reindex(const int8_t *q_idx, const int8_t *k_idx, const float *k_scale,
                                  const int32_t *pool, const int64_t *ctx_len,
                                  const int64_t *q_pos, int B, int Nq, int H, int D, int64_t cap,
                                  int P, float *pool_score, int32_t *pool_pos, void *stream) {
    int st = check_indexer_common(q_idx, k_idx, k_scale, ctx_len, B, Nq, H, D, cap);
    if (st) return st;
    if (!pool || !pool_score || !pool_pos) return CSA2_ERR_NULL;
    if (P < 0 || P > (1 << 24)) return CSA2_ERR_SHAPE;
    if ((int64_t)B * Nq * P == 0) return CSA2_OK;
    ReindexArgs a{q_idx, k_idx, k_scale, pool, ctx_len, q_pos, B, Nq, H * D, P, cap,
                  pool_score, pool_pos, nullptr};
    return dispatch_reindex(a, (cudaStream_t)stream, false);
}

extern "C" int csa2_pool_gather(const float *tok_score, const int32_t *pool,
                                const int64_t *ctx_len, const int64_t *q_pos, int B, int Nq, int P,
                                int64_t cap, float *pool_score, int32_t *pool_pos, void *stream) {
    if (!tok_score || !pool || !ctx_len || !pool_score || !pool_pos) return CSA2_ERR_NULL;
    if (B < 0 || Nq < 0 || P < 0 || P > (1 << 24) || cap < 1) return CSA2_ERR_SHAPE;
    const int64_t total = (int64_t)B * Nq * P * 8;
    if (total == 0) return CSA2_OK;
    const int T = 256;
    const int64_t g = (total + T - 1) / T;
    if (g > INT32_MAX) return CSA2_ERR_SHAPE;
    pool_gather_kernel<<<(unsigned)g, T, 0, (cudaStream_t)stream>>>(tok_score, pool, ctx_len, q_pos,
                                                                   B, Nq, P, cap, pool_score,
                                                                   pool_pos, nullptr);
    return launch_status();
}

namespace csa2 {

int launch_index_full_hist(const int8_t *q_idx, const int8_t *k_idx, const float *k_scale,
                           const int64_t *ctx_len, int B, int H, int D, int64_t cap,
                           float *tok_score, float *blk_score, int32_t *n_blk, uint32_t *hist,
                           cudaStream_t s) {
    ScanArgs a{q_idx, k_idx, k_scale, ctx_len, nullptr, B, 1, H * D, cap, (cap + 7) / 8,
               tok_score, blk_score, n_blk, hist};
    return dispatch_scan(a, s, true);
}

int launch_pool_gather_hist(const float *tok_score, const int32_t *pool, const int64_t *ctx_len,
                            int B, int P, int64_t cap, float *pool_score, int32_t *pool_pos,
                            uint32_t *hist, cudaStream_t s) {
    const int64_t total = (int64_t)B * P * 8;
    if (total == 0) return CSA2_OK;
    const int T = 256;
    return launch_kernel(true, pool_gather_kernel, dim3((unsigned)((total + T - 1) / T)), dim3(T), 0,
                         s, tok_score, pool, ctx_len, nullptr, B, 1, P, cap, pool_score, pool_pos,
                         hist);
}

int launch_reindex_hist(const int8_t *q_idx, const int8_t *k_idx, const float *k_scale,
                        const int32_t *pool, const int64_t *ctx_len, int B, int H, int D,
                        int64_t cap, int P, float *pool_score, int32_t *pool_pos, uint32_t *hist,
                        cudaStream_t s) {
    ReindexArgs a{q_idx, k_idx, k_scale, pool, ctx_len, nullptr, B, 1, H * D, P, cap,
                  pool_score, pool_pos, hist};
    return dispatch_reindex(a, s, true);
}

}  // namespace csa2
