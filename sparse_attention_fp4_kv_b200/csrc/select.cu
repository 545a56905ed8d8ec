// Full-layer selection of one query in one CTA: the pool of blocks and the
// top-k tokens of the pool, from the scan's block and token scores.
//
// "DeepSeek V4.1 Flash KV Cache: 890 Bytes per Token Explained", indexer
// section: the pool keeps the best 2,048 blocks of 8 tokens and each query
// keeps its best 512 candidates. "DeepSeek-V4.1-Flash: 890 Bytes Per Token,
// 437x Smaller KV Cache", CSA2 section: a Full layer builds the pool and
// selects a fresh top-512.
//
// The same result as three calls (block top-k, pool gather, token top-k) with
// nothing written to global memory between them: for rows that fit in shared
// memory (at most 16,384 blocks and 16,384 pooled tokens), one CTA per query
//   1. loads the block scores as 32-bit order keys and selects the best P by
//      (score desc, block asc): radix digits below the bits that every key of
//      the row shares (so the first histogram spreads), then a tie rank in
//      index order; writes the pool (ascending block ids);
//   2. selects the best K blocks the same way (K <= P): every one of the best
//      K tokens lies in one of them, since each block ranked ahead of a token's
//      block holds its own maximum, a token ranked ahead of it;
//   3. gathers those blocks' token scores (positions below the query's visible
//      length) into the key array, in position order, and selects the best K
//      tokens, written as ascending positions.
// Key 0 marks a slot that holds no candidate (no finite score maps to 0).
// Emission walks each warp's contiguous range with ballots, so the output is
// in index order without a sort.
#include "common.cuh"

namespace csa2 {

constexpr int FS_THREADS = 512;
constexpr int FS_WARPS = FS_THREADS / 32;
constexpr int FS_MAXN = 16384;  // keys held in shared memory
constexpr int FS_HIST = 4096;
// Histogram bin b lives at b + b / 32: a thread scanning its run of
// consecutive bins then hits a different bank from every other lane.
__device__ __forceinline__ int hpad(int b) { return b + (b >> 5); }
constexpr int FS_HIST_WORDS = FS_HIST + FS_HIST / 32;

struct FsState {
    uint32_t wsum[32];
    int digit;
    uint32_t above, match, total;
    uint32_t wcnt[FS_WARPS];  // packed (greater << 16 | equal) counts per warp
    uint32_t wor[FS_WARPS], wand[FS_WARPS], wn[FS_WARPS];
};

// Bin d where the count of keys in bins >= d first reaches kk (scanning from
// the top bin); st.above = keys in bins above d, st.match = keys in d,
// st.total = all counted keys.
__device__ void fs_find_digit(const uint32_t *hist, int NB, int kk, FsState &st) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int BPT = (NB + FS_THREADS - 1) / FS_THREADS;
    const int b0 = tid * BPT;
    uint32_t local = 0;
    for (int j = 0; j < BPT; j++)
        if (b0 + j < NB) local += hist[hpad(b0 + j)];
    uint32_t x = local;  // inclusive suffix sum within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
    }
    if (lane == 0) st.wsum[warp] = x;
    __syncthreads();
    uint32_t warps_above = 0, all = 0;
    for (int w = 0; w < FS_WARPS; w++) {
        all += st.wsum[w];
        if (w > warp) warps_above += st.wsum[w];
    }
    uint32_t above = (x - local) + warps_above;
    for (int j = BPT - 1; j >= 0; j--) {
        const int bin = b0 + j;
        if (bin >= NB) continue;
        const uint32_t h = hist[hpad(bin)];
        if (above < (uint32_t)kk && above + h >= (uint32_t)kk) {
            st.digit = bin;
            st.above = above;
            st.match = h;
        }
        above += h;
    }
    if (tid == 0) st.total = all;
    __syncthreads();
}

// The k best of keys[0..n) by (key desc, index asc), as a threshold: every
// key > T is selected, and of the keys == T the first `take` in index order.
// T = 0 (take = 0) when all candidates are selected. Returns the number
// selected. The digits start below the leading bits that all candidate keys
// share (an OR / AND reduction), 12 bits first, then 10 at a time.
// With k2 > 0 (k2 <= k), C2 also receives a key value that every one of the
// best k2 keys reaches, from the first digit's histogram: the keys >= C2 are a
// superset of the best k2 (the rest of their first-digit bin included).
__device__ int fs_select(const uint32_t *keys, int n, int k, uint32_t *hist, FsState &st,
                         uint32_t &T, int &take, int k2, uint32_t &C2) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t kor = 0, kand = 0xFFFFFFFFu, cnt = 0;
    for (int i = tid; i < n; i += FS_THREADS) {
        const uint32_t key = keys[i];
        if (key) {
            kor |= key;
            kand &= key;
            cnt++;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kor |= __shfl_xor_sync(0xffffffffu, kor, o);
        kand &= __shfl_xor_sync(0xffffffffu, kand, o);
        cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    }
    if (lane == 0) {
        st.wor[warp] = kor;
        st.wand[warp] = kand;
        st.wn[warp] = cnt;
    }
    __syncthreads();
    kor = 0;
    kand = 0xFFFFFFFFu;
    cnt = 0;
    for (int w = 0; w < FS_WARPS; w++) {
        kor |= st.wor[w];
        kand &= st.wand[w];
        cnt += st.wn[w];
    }
    C2 = 1u;  // every candidate (key 0 is no candidate)
    if (cnt <= (uint32_t)k) {
        T = 0;
        take = 0;
        return (int)cnt;
    }
    // the candidates share their top L bits; all of them equal when L = 32
    const int L = __clz(kor ^ kand);
    if (L == 32) {
        T = kand;
        take = k;
        C2 = kand;
        return k;
    }
    int shift = 32 - L > 12 ? 32 - L - 12 : 0;
    int nbits = 32 - L - shift;
    uint32_t prefix = L == 0 ? 0u : (kand >> (32 - L));  // the matched high bits
    int pshift = 32 - L;
    int kk = k;
#pragma unroll 1
    while (true) {
        const uint32_t mask = (1u << nbits) - 1u;
        for (int b = tid; b <= (int)mask; b += FS_THREADS) hist[hpad(b)] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += FS_THREADS) {
            const uint32_t key = keys[i];
            if (key && (pshift >= 32 || (key >> pshift) == prefix))
                atomicAdd(&hist[hpad((int)((key >> shift) & mask))], 1u);
        }
        __syncthreads();
        if (k2 > 0 && pshift == 32 - L) {
            // first digit: the bin of the k2-th best key (all keys share the
            // top L bits, so the bin's lowest key value bounds the best k2)
            fs_find_digit(hist, (int)mask + 1, k2, st);
            const uint32_t c = ((prefix << nbits) | (uint32_t)st.digit) << shift;
            C2 = c ? c : 1u;
        }
        fs_find_digit(hist, (int)mask + 1, kk, st);
        prefix = (prefix << nbits) | (uint32_t)st.digit;
        kk -= (int)st.above;
        if (shift == 0) break;
        pshift = shift;
        nbits = shift > 10 ? 10 : shift;
        shift -= nbits;
        __syncthreads();
    }
    T = prefix;
    take = kk;
    return k;
}

// Calls f(out_slot, index) for the selected keys (key(i), i < n) in
// ascending index order. Warp w walks the contiguous range [w R, w R + R),
// 32 keys per step.
template <typename KeyF, typename F>
__device__ void fs_emit(KeyF key_of, int n, uint32_t T, int take, FsState &st, F f) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int R = ((n + FS_WARPS * 32 - 1) / (FS_WARPS * 32)) * 32;
    const int i0 = warp * R;
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t gt = 0, eq = 0;
    for (int j = i0; j < i0 + R && j < n; j += 32) {
        const int i = j + lane;
        const uint32_t key = i < n ? key_of(i) : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, key > T));
        eq += __popc(__ballot_sync(0xffffffffu, key != 0 && key == T));
    }
    if (lane == 0) st.wcnt[warp] = (gt << 16) | eq;
    __syncthreads();
    uint32_t gt_base = 0, eq_base = 0;
    for (int w = 0; w < warp; w++) {
        gt_base += st.wcnt[w] >> 16;
        eq_base += st.wcnt[w] & 0xFFFFu;
    }
    for (int j = i0; j < i0 + R && j < n; j += 32) {
        const int i = j + lane;
        const uint32_t key = i < n ? key_of(i) : 0u;
        const bool g = key > T;
        const bool e = key != 0 && key == T;
        const uint32_t bg = __ballot_sync(0xffffffffu, g);
        const uint32_t be = __ballot_sync(0xffffffffu, e);
        const uint32_t erank = eq_base + __popc(be & lt_mask);
        const bool sel = g || (e && erank < (uint32_t)take);
        // ties taken before this lane: min(take, eq rank) over the eq keys so far
        const uint32_t eq_taken_before =
            min((uint32_t)take, eq_base + __popc(be & lt_mask));
        if (sel) f((int)(gt_base + __popc(bg & lt_mask) + eq_taken_before), i);
        gt_base += __popc(bg);
        eq_base += __popc(be);
    }
    __syncthreads();
}

__global__ void __launch_bounds__(FS_THREADS, 3) full_select_kernel(
    const float *__restrict__ blk, const int32_t *__restrict__ n_blk, const float *__restrict__ tok,
    const int64_t *ctx_len, const int64_t *q_pos, int B, int Nq, int64_t cap, int P, int K,
    int32_t *__restrict__ pool, int32_t *__restrict__ top) {
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int64_t nkeys = (cap + 7) / 8 > 8 * (int64_t)(K < P ? K : P) ? (cap + 7) / 8
                                                                       : 8 * (int64_t)(K < P ? K : P);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw);  // [nkeys]
    uint32_t *hist = keys + nkeys;                             // [FS_HIST_WORDS]
    int32_t *pool_s = reinterpret_cast<int32_t *>(hist + FS_HIST_WORDS);  // [P]
    int32_t *kblk_s = pool_s + P;                                    // [P]
    __shared__ FsState st;
    const int tid = threadIdx.x;
    const int64_t row = blockIdx.x;
    const int b = (int)(row / Nq), qi = (int)(row % Nq);
    const int64_t nblk_cap = (cap + 7) / 8;
    int64_t V = visible_len(ctx_len, q_pos, b, qi, Nq);
    if (V > cap) V = cap;
    int nb = n_blk[row];
    nb = nb < 0 ? 0 : (nb > nblk_cap ? (int)nblk_cap : nb);

    // ---- 1. pool: the best P blocks
    const float *brow = blk + row * nblk_cap;
    for (int i0 = 0; i0 < nb; i0 += FS_THREADS * 8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int i = i0 + u * FS_THREADS + tid;
            v[u] = i < nb ? __ldg(brow + i) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int i = i0 + u * FS_THREADS + tid;
            if (i < nb) keys[i] = f32_order_key(v[u]);
        }
    }
    __syncthreads();
    uint32_t T, C2;
    int take;
    const int npool = fs_select(keys, nb, P, hist, st, T, take, K < P ? K : 0, C2);
    fs_emit([&](int i) { return keys[i]; }, nb, T, take, st, [&](int slot, int i) { pool_s[slot] = i; });
    int32_t *prow = pool + row * P;
    for (int s = tid; s < P; s += FS_THREADS) {
        if (s >= npool) pool_s[s] = -1;
        prow[s] = pool_s[s];
    }
    __syncthreads();

    // ---- 2. blocks whose tokens are candidates (ascending): the pooled blocks
    // whose key reaches C2, a superset of the best K blocks, when their tokens
    // fit the key array; else exactly the best K blocks
    const int32_t *kblk = pool_s;
    int nkb = npool;
    if (K < npool) {
        int n_c2 = 0;
        for (int s0 = 0; s0 < npool; s0 += FS_THREADS)
            n_c2 += __syncthreads_count(s0 + tid < npool && keys[pool_s[s0 + tid]] >= C2);
        if (8 * (int64_t)n_c2 <= nkeys) {
            fs_emit([&](int s) { return keys[pool_s[s]]; }, npool, C2 - 1u, 0, st,
                    [&](int slot, int s) { kblk_s[slot] = pool_s[s]; });
            nkb = n_c2;
        } else {
            uint32_t unused;
            fs_select(keys, nb, K, hist, st, T, take, 0, unused);
            fs_emit([&](int s) { return keys[pool_s[s]]; }, npool, T, take, st,
                    [&](int slot, int s) { kblk_s[slot] = pool_s[s]; });
            nkb = K;
        }
        kblk = kblk_s;
    }

    // ---- 3. their token scores in position order, then the best K tokens
    const float *trow = tok + row * cap;
    const int n2 = 8 * nkb;
    for (int i0 = 0; i0 < n2; i0 += FS_THREADS * 8) {
        float v[8];
        bool ok[8];
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int i = i0 + u * FS_THREADS + tid;
            const int32_t j = i < n2 ? kblk[i >> 3] : -1;
            const int64_t p = 8 * (int64_t)j + (i & 7);
            ok[u] = j >= 0 && p < V;
            v[u] = ok[u] ? __ldg(trow + p) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int i = i0 + u * FS_THREADS + tid;
            if (i < n2) keys[i] = ok[u] ? f32_order_key(v[u]) : 0u;
        }
    }
    __syncthreads();
    uint32_t unused;
    const int ntop = fs_select(keys, n2, K, hist, st, T, take, 0, unused);
    int32_t *trow_out = top + row * K;
    fs_emit([&](int i) { return keys[i]; }, n2, T, take, st,
            [&](int slot, int i) { trow_out[slot] = 8 * kblk[i >> 3] + (i & 7); });
    for (int s = ntop + tid; s < K; s += FS_THREADS) trow_out[s] = -1;
}

// key array (the larger of the block row and the gathered tokens), the
// histogram, the pool and the best blocks
size_t full_select_smem(int64_t cap, int P, int K) {
    const int64_t nb = (cap + 7) / 8;
    const int64_t n2 = 8 * (int64_t)(K < P ? K : P);
    const int64_t nkeys = nb > n2 ? nb : n2;
    return (size_t)(nkeys + FS_HIST_WORDS) * 4 + (size_t)P * 8;
}

bool full_select_supported(int64_t cap, int P, int K) {
    return (cap + 7) / 8 <= FS_MAXN && P >= 1 && 8 * (int64_t)P <= FS_MAXN && K >= 1 && K <= 8 * P;
}

int launch_full_select(const float *blk, const int32_t *n_blk, const float *tok,
                       const int64_t *ctx_len, const int64_t *q_pos, int B, int Nq, int64_t cap,
                       int P, int K, int32_t *pool, int32_t *top, cudaStream_t s, bool pdl) {
    const int64_t rows = (int64_t)B * Nq;
    if (rows == 0) return CSA2_OK;
    if (rows > INT32_MAX) return CSA2_ERR_SHAPE;
    const size_t smem = full_select_smem(cap, P, K);
    static PerDevice attrs_set;
    // two CTAs per SM: dynamic shared memory up to the largest row, and the
    // largest shared-memory carveout
    if (attrs_set.get([] {
            return cudaFuncSetAttribute(full_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)full_select_smem(8 * (int64_t)FS_MAXN, kPoolBlocks,
                                                              kPoolBlocks)) == cudaSuccess &&
                           cudaFuncSetAttribute(full_select_kernel,
                                                cudaFuncAttributePreferredSharedMemoryCarveout,
                                                (int)cudaSharedmemCarveoutMaxShared) == cudaSuccess
                       ? 1
                       : -1;
        }) < 0)
        return CSA2_ERR_CUDA;
    return launch_kernel(pdl, full_select_kernel, dim3((unsigned)rows), dim3(FS_THREADS), smem, s,
                         blk, n_blk, tok, ctx_len, q_pos, B, Nq, cap, P, K, pool, top);
}

}  // namespace csa2

using namespace csa2;

extern "C" int csa2_full_select(const float *blk_score, const int32_t *n_blk,
                                const float *tok_score, const int64_t *ctx_len,
                                const int64_t *q_pos, int B, int Nq, int64_t cap, int P, int K,
                                int32_t *pool, int32_t *top, void *stream) {
    if (!blk_score || !n_blk || !tok_score || !ctx_len || !pool || !top) return CSA2_ERR_NULL;
    if (B < 0 || Nq < 0 || cap < 1) return CSA2_ERR_SHAPE;
    if (P < 1 || P > kPoolBlocks || !full_select_supported(cap, P, K)) return CSA2_ERR_SHAPE;
    return launch_full_select(blk_score, n_blk, tok_score, ctx_len, q_pos, B, Nq, cap, P, K, pool,
                              top, (cudaStream_t)stream, false);
}
