// Deterministic top-k selection (pool of blocks, top-512 tokens).
//
// "DeepSeek V4.1 Flash KV Cache: 890 Bytes per Token Explained", indexer
// section: the pool keeps the best 2,048 blocks of 8 tokens and each query
// keeps its best 512 candidates. "DeepSeek-V4.1-Flash: 890 Bytes Per Token,
// 437x Smaller KV Cache", CSA2 section: Full and Reindex layers select a fresh
// top-512.
//
// Every candidate gets a unique 64-bit key: the order-preserving bits of its
// fp32 score above the bit-inverted position, so "higher key" means "higher
// score, then lower position" and there are no ties. The k-th largest key is
// found by MSB-first radix selection: a 12-bit digit first (sign, exponent and
// three mantissa bits), then 8-bit digits. The digit passes read the row from
// global memory (L2) until the candidates that share the current prefix fit in
// shared memory; one more pass moves those into shared memory and sends every
// candidate above the prefix straight to the output list; the remaining digits
// run in shared memory. The selected positions are sorted ascending with a
// bitonic sort. One CTA of 1024 threads per row; no global scratch.
#include "common.cuh"

namespace csa2 {

constexpr int TK_THREADS = 1024;
constexpr int TK_BUF = 8192;   // shared-memory candidate buffer (64-bit keys)
constexpr int TK_MAXK = 4096;  // largest k
constexpr int TK_HIST = 4096;  // bins of the first digit
constexpr size_t TK_SMEM = TK_HIST * 4 + TK_BUF * 8 + TK_MAXK * 4;

struct TopkArgs {
    const float *score;
    const int32_t *cand_pos;
    const int32_t *n_valid;
    int R;
    int64_t n;
    int k;
    int32_t *out;
};

__device__ __forceinline__ bool aligned16(const void *p) {
    return (reinterpret_cast<uintptr_t>(p) & 15) == 0;
}

struct TopkShared {
    uint32_t *hist;
    uint64_t *buf;
    int32_t *sel;
};

struct TopkState {
    uint64_t prefix, mask;
    int kk;           // rank still to find inside the prefix group
    int digit;        // digit found by the last pass
    uint32_t above;   // candidates above the digit inside the prefix group
    uint32_t match;   // candidates with the digit inside the prefix group
    uint32_t total;   // candidates counted by the last pass
    int nsel, nbuf;
    uint32_t wsum[32];
};

// Block-wide (NT threads): given hist[0..NB), find the bin d where the count
// of keys at or above it first reaches kk (scanning from the top bin down).
// Thread t sums the contiguous bins [t BPT, t BPT + BPT); with 4 bins per
// thread it reads them with one 16-byte load (a warp's loads are then
// conflict-free) and keeps them in registers for the second walk.
template <int NT = TK_THREADS>
__device__ void find_digit(const uint32_t *hist, int NB, int kk, TopkState &st) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int BPT = (NB + NT - 1) / NT;
    const int b0 = tid * BPT;
    const bool quad = NB == 4 * NT;
    uint4 q4 = make_uint4(0, 0, 0, 0);
    uint32_t local = 0;
    if (quad) {
        q4 = reinterpret_cast<const uint4 *>(hist)[tid];
        local = q4.x + q4.y + q4.z + q4.w;
    } else {
        for (int j = 0; j < BPT; j++)
            if (b0 + j < NB) local += hist[b0 + j];
    }
    // inclusive suffix sum inside the warp
    uint32_t x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
    }
    if (lane == 0) st.wsum[warp] = x;
    __syncthreads();
    uint32_t warps_above = 0, all = 0;
    for (int w = 0; w < NT / 32; w++) {
        all += st.wsum[w];
        if (w > warp) warps_above += st.wsum[w];
    }
    uint32_t above = (x - local) + warps_above;  // keys in bins above my bins
    for (int j = BPT - 1; j >= 0; j--) {
        const int bin = b0 + j;
        if (bin >= NB) continue;
        const uint32_t h = quad ? (j == 3 ? q4.w : j == 2 ? q4.z : j == 1 ? q4.y : q4.x) : hist[bin];
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

// find_digit over a producer's 4096-bin first-digit histogram row in global
// memory, without a shared-memory copy: thread t loads its TK_HIST / NT
// contiguous bins straight into registers (16-byte loads).
template <int NT>
__device__ void hist_threshold(const uint32_t *gh, int kk, TopkState &st) {
    constexpr int BPT = TK_HIST / NT;
    static_assert(BPT % 4 == 0 && BPT * NT == TK_HIST, "whole 16-byte groups per thread");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t hb[BPT];
    const uint4 *hp = reinterpret_cast<const uint4 *>(gh) + (BPT / 4) * tid;
#pragma unroll
    for (int q = 0; q < BPT / 4; q++) {
        const uint4 v = hp[q];
        hb[4 * q] = v.x;
        hb[4 * q + 1] = v.y;
        hb[4 * q + 2] = v.z;
        hb[4 * q + 3] = v.w;
    }
    uint32_t local = 0;
#pragma unroll
    for (int j = 0; j < BPT; j++) local += hb[j];
    uint32_t x = local;  // inclusive suffix sum over the lanes of the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
    }
    if (lane == 0) st.wsum[warp] = x;
    __syncthreads();
    uint32_t above = x - local, total = 0;
    for (int w = 0; w < NT / 32; w++) {
        total += st.wsum[w];
        if (w > warp) above += st.wsum[w];
    }
#pragma unroll
    for (int j = BPT - 1; j >= 0; j--) {
        if (above < (uint32_t)kk && above + hb[j] >= (uint32_t)kk) {
            st.digit = BPT * tid + j;
            st.above = above;
            st.match = hb[j];
        }
        above += hb[j];
    }
    if (tid == 0) st.total = total;
    __syncthreads();
}

// hist_threshold for rank k1 (into st) and, from the same registers, the bin
// of rank k2 into *d2 (-1 when the row holds at most k2 keys): one read of the
// histogram row for both.
template <int NT>
__device__ void hist_threshold2(const uint32_t *gh, int k1, int k2, TopkState &st, int *d2) {
    constexpr int BPT = TK_HIST / NT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t hb[BPT];
    const uint4 *hp = reinterpret_cast<const uint4 *>(gh) + (BPT / 4) * tid;
#pragma unroll
    for (int q = 0; q < BPT / 4; q++) {
        const uint4 v = hp[q];
        hb[4 * q] = v.x;
        hb[4 * q + 1] = v.y;
        hb[4 * q + 2] = v.z;
        hb[4 * q + 3] = v.w;
    }
    uint32_t local = 0;
#pragma unroll
    for (int j = 0; j < BPT; j++) local += hb[j];
    uint32_t x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
    }
    if (lane == 0) st.wsum[warp] = x;
    if (tid == 0) *d2 = -1;
    __syncthreads();
    uint32_t above = x - local, total = 0;
    for (int w = 0; w < NT / 32; w++) {
        total += st.wsum[w];
        if (w > warp) above += st.wsum[w];
    }
#pragma unroll
    for (int j = BPT - 1; j >= 0; j--) {
        if (above < (uint32_t)k1 && above + hb[j] >= (uint32_t)k1) {
            st.digit = BPT * tid + j;
            st.above = above;
            st.match = hb[j];
        }
        if (total > (uint32_t)k2 && above < (uint32_t)k2 && above + hb[j] >= (uint32_t)k2) *d2 = BPT * tid + j;
        above += hb[j];
    }
    if (tid == 0) st.total = total;
    __syncthreads();
}

// Candidate i of row r from global memory; false if it is not a candidate.
__device__ __forceinline__ bool load_cand(const TopkArgs &a, int64_t r, int64_t i, uint64_t &key) {
    const int32_t pos = a.cand_pos ? a.cand_pos[r * a.n + i] : (int32_t)i;
    key = rank_key(a.score[r * a.n + i], pos);
    return pos >= 0;
}

constexpr int TK_UNROLL = 4;  // 16-byte loads in flight per thread

// Four consecutive candidates i0..i0+3 (i0 % 4 == 0) with 16-byte loads when the
// row is 16-byte aligned, else element by element.
__device__ __forceinline__ void load_cand4(const TopkArgs &a, int64_t r, int64_t i0, int64_t nv,
                                           bool vec, uint64_t (&key)[4], bool (&ok)[4]) {
    if (vec && i0 + 3 < nv) {
        const float4 s = *reinterpret_cast<const float4 *>(a.score + r * a.n + i0);
        int4 p = make_int4((int)i0, (int)i0 + 1, (int)i0 + 2, (int)i0 + 3);
        if (a.cand_pos) p = *reinterpret_cast<const int4 *>(a.cand_pos + r * a.n + i0);
        key[0] = rank_key(s.x, p.x);
        key[1] = rank_key(s.y, p.y);
        key[2] = rank_key(s.z, p.z);
        key[3] = rank_key(s.w, p.w);
        ok[0] = p.x >= 0;
        ok[1] = p.y >= 0;
        ok[2] = p.z >= 0;
        ok[3] = p.w >= 0;
    } else {
#pragma unroll
        for (int u = 0; u < 4; u++) ok[u] = (i0 + u < nv) && load_cand(a, r, i0 + u, key[u]);
    }
}

// Calls f(key) for every candidate of row r (i < nv), TK_UNROLL x 4 per thread
// per iteration.
template <typename F>
__device__ __forceinline__ void for_each_cand(const TopkArgs &a, int64_t r, int64_t nv, bool vec,
                                              F f) {
    const int64_t step = (int64_t)TK_THREADS * 4 * TK_UNROLL;
    for (int64_t b0 = 0; b0 < nv; b0 += step) {
        uint64_t key[TK_UNROLL][4];
        bool ok[TK_UNROLL][4];
#pragma unroll
        for (int u = 0; u < TK_UNROLL; u++)
            load_cand4(a, r, b0 + ((int64_t)u * TK_THREADS + threadIdx.x) * 4, nv, vec, key[u],
                       ok[u]);
#pragma unroll
        for (int u = 0; u < TK_UNROLL; u++)
#pragma unroll
            for (int v = 0; v < 4; v++)
                if (ok[u][v]) f(key[u][v]);
    }
}

// One digit histogram pass over the global row: keys whose masked bits equal
// the prefix are binned by (key >> shift) & (NB - 1).
__device__ void global_hist_pass(const TopkArgs &a, int64_t r, int64_t nv, bool vec,
                                 uint32_t *hist, int NB, int shift, uint64_t prefix,
                                 uint64_t mask) {
    for (int b = threadIdx.x; b < NB; b += TK_THREADS) hist[b] = 0;
    __syncthreads();
    for_each_cand(a, r, nv, vec, [&](uint64_t key) {
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (uint64_t)(NB - 1)], 1u);
    });
    __syncthreads();
}

template <int NT = TK_THREADS>
__device__ void smem_hist_pass(const uint64_t *buf, int nbuf, uint32_t *hist, int NB, int shift,
                               uint64_t prefix, uint64_t mask) {
    for (int b = threadIdx.x; b < NB; b += NT) hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < nbuf; i += NT) {
        const uint64_t key = buf[i];
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (uint64_t)(NB - 1)], 1u);
    }
    __syncthreads();
}

// Ascending bitonic sort of v[0..n) (n <= TK_MAXK) padded to a power of two.
__device__ void bitonic_sort_asc(int32_t *v, int n) {
    int N = 1;
    while (N < n) N <<= 1;
    for (int i = n + threadIdx.x; i < N; i += TK_THREADS) v[i] = INT32_MAX;
    __syncthreads();
    for (int size = 2; size <= N; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = threadIdx.x; t < N / 2; t += TK_THREADS) {
                const int lo = 2 * t - (t & (stride - 1));
                const int hi = lo + stride;
                const bool up = ((lo & size) == 0);
                const int32_t x = v[lo], y = v[hi];
                if ((x > y) == up) {
                    v[lo] = y;
                    v[hi] = x;
                }
            }
            __syncthreads();
        }
    }
}

__device__ __forceinline__ TopkShared topk_shared(uint8_t *smem_raw) {
    return TopkShared{reinterpret_cast<uint32_t *>(smem_raw),
                      reinterpret_cast<uint64_t *>(smem_raw + TK_HIST * 4),
                      reinterpret_cast<int32_t *>(smem_raw + TK_HIST * 4 + TK_BUF * 8)};
}

// The whole selection of row r by one CTA of TK_THREADS threads.
__device__ void topk_row_full(const TopkArgs &a, int64_t r, TopkShared sh, TopkState &st) {
    int64_t nv = a.n;
    if (a.n_valid) {
        const int64_t v = a.n_valid[r];
        nv = v < 0 ? 0 : (v < a.n ? v : a.n);
    }
    const bool vec = ((r * a.n) % 4 == 0) && aligned16(a.score) &&
                     (a.cand_pos == nullptr || aligned16(a.cand_pos));
    if (threadIdx.x == 0) {
        st.prefix = 0;
        st.mask = 0;
        st.kk = a.k;
        st.nsel = 0;
        st.nbuf = 0;
    }
    __syncthreads();

    // ---- digit passes over the global row
    int shift = 52, NB = TK_HIST;
    bool all_selected = false, exact = false;
    while (true) {
        global_hist_pass(a, r, nv, vec, sh.hist, NB, shift, st.prefix, st.mask);
        if (shift == 52) {
            find_digit(sh.hist, NB, st.kk, st);
            if (st.total <= (uint32_t)a.k) {  // every candidate is selected
                all_selected = true;
                break;
            }
        } else {
            find_digit(sh.hist, NB, st.kk, st);
        }
        if (threadIdx.x == 0) {
            st.kk -= (int)st.above;
            st.prefix |= (uint64_t)st.digit << shift;
            st.mask |= (uint64_t)(NB - 1) << shift;
        }
        __syncthreads();
        if (st.match == (uint32_t)st.kk || shift == 0) {
            exact = true;  // the whole prefix group is selected
            break;
        }
        if (st.match <= (uint32_t)TK_BUF) break;
        const int next = shift >= 8 ? 8 : shift;
        shift -= next;
        NB = 1 << next;
    }

    const uint64_t gprefix = st.prefix, gmask = st.mask;
    // ---- one pass: select everything above the prefix group; keep the group
    for_each_cand(a, r, nv, vec, [&](uint64_t key) {
        const uint64_t km = key & gmask;
        if (all_selected || km > gprefix || (exact && km == gprefix)) {
            const int s = atomicAdd(&st.nsel, 1);
            if (s < TK_MAXK) sh.sel[s] = rank_key_pos(key);
        } else if (km == gprefix) {
            const int s = atomicAdd(&st.nbuf, 1);
            if (s < TK_BUF) sh.buf[s] = key;
        }
    });
    __syncthreads();

    // ---- remaining digits inside shared memory
    if (!all_selected && !exact) {
        const int nbuf = min(st.nbuf, TK_BUF);
        while (true) {
            const int next = shift >= 8 ? 8 : shift;
            shift -= next;
            NB = 1 << next;
            smem_hist_pass(sh.buf, nbuf, sh.hist, NB, shift, st.prefix, st.mask);
            find_digit(sh.hist, NB, st.kk, st);
            if (threadIdx.x == 0) {
                st.kk -= (int)st.above;
                st.prefix |= (uint64_t)st.digit << shift;
                st.mask |= (uint64_t)(NB - 1) << shift;
            }
            __syncthreads();
            if (st.match == (uint32_t)st.kk || shift == 0) break;
        }
        const uint64_t p = st.prefix, m = st.mask;
        for (int i = threadIdx.x; i < nbuf; i += TK_THREADS) {
            const uint64_t key = sh.buf[i];
            if ((key & m) >= p && (key & gmask) == gprefix) {
                const int s = atomicAdd(&st.nsel, 1);
                if (s < TK_MAXK) sh.sel[s] = rank_key_pos(key);
            }
        }
        __syncthreads();
    }

    const int nsel = min(st.nsel, a.k);
    bitonic_sort_asc(sh.sel, nsel);
    int32_t *out = a.out + r * a.k;
    for (int i = threadIdx.x; i < a.k; i += TK_THREADS) out[i] = i < nsel ? sh.sel[i] : -1;
}

__global__ void __launch_bounds__(TK_THREADS, 1) topk_kernel(TopkArgs a) {
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ TopkState st;
    topk_row_full(a, blockIdx.x, topk_shared(smem_raw), st);
}

// ------------------------------------------------------------------ histogram-fed selection
// Used inside the decode step, where every candidate list is in ascending
// position order (block ids, or the pool's blocks expanded to tokens): there,
// "lower position" equals "lower candidate index", so the ranking key can
// carry the index instead of the position, and the output (ascending
// positions) is the selected indices in index order.
//
// The producer of the scores (scan, pool gather, Reindex) has already counted
// every candidate of row r into hist[r][top 12 bits of its key]. From the
// histogram, the compaction kernel (many CTAs per row) sends the index of
// every candidate above the threshold bin straight to the selection and the
// threshold bin's keys to a tie list (one atomic per warp per list); the
// finish kernel (one CTA per row) resolves the tie list in shared memory,
// marks the selected indices in a bitmap and writes them in index order via a
// block-wide prefix count, and clears the row's histogram and counters for the
// next producer. A tie list longer than its buffer falls back to the whole
// single-CTA selection of the row.
constexpr int TC_THREADS = 256;
constexpr int TC_SLICE = 4096;  // candidates per compaction CTA
constexpr int TC_PER = TC_SLICE / TC_THREADS;
constexpr int64_t TF_MAX_N = (int64_t)TK_BUF * 2 * 32;  // bitmap capacity of the finish

struct TopkHistWs {
    uint32_t *hist;  // [R][4096]
    int *cnt;        // [R][4]: selected, ties, CTAs done (fused compaction), unused
    int32_t *sel;    // [R][k] candidate indices
    uint64_t *tie;   // [R][TK_BUF] keys
};

// Copy n elements of T from global to shared memory, 8 loads in flight per thread.
template <typename T>
__device__ __forceinline__ void load_batched(T *dst, const T *src, int n) {
    for (int i0 = 0; i0 < n; i0 += 8 * TK_THREADS) {
        T v[8];
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int i = i0 + u * TK_THREADS + threadIdx.x;
            if (i < n) v[u] = src[i];
        }
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int i = i0 + u * TK_THREADS + threadIdx.x;
            if (i < n) dst[i] = v[u];
        }
    }
}

__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

__global__ void __launch_bounds__(TC_THREADS) topk_compact_kernel(TopkArgs a, TopkHistWs ws) {
    grid_dep_wait();
    grid_dep_launch();
    __shared__ TopkState st;
    const int64_t r = blockIdx.y;
    int64_t nv = a.n;
    if (a.n_valid) {
        const int64_t v = a.n_valid[r];
        nv = v < 0 ? 0 : (v < a.n ? v : a.n);
    }
    const int64_t i_beg = (int64_t)blockIdx.x * TC_SLICE;
    if (i_beg >= nv) return;
    hist_threshold<TC_THREADS>(ws.hist + r * TK_HIST, a.k, st);
    const bool all = st.total <= (uint32_t)a.k;
    const uint64_t d = (uint64_t)st.digit;
    const bool vec = ((r * a.n) % 4 == 0) && aligned16(a.score) &&
                     (a.cand_pos == nullptr || aligned16(a.cand_pos));
    uint64_t key[TC_PER];
    uint32_t selm = 0, tiem = 0;
#pragma unroll
    for (int u = 0; u < TC_PER / 4; u++) {
        const int64_t i0 = i_beg + 4 * ((int64_t)u * TC_THREADS + threadIdx.x);
        uint64_t pk[4];
        bool ok[4];
        load_cand4(a, r, i0, nv, vec, pk, ok);
#pragma unroll
        for (int v = 0; v < 4; v++) {
            const int j = 4 * u + v;
            // index-keyed: the ordered score bits above the inverted index
            key[j] = (pk[v] & 0xFFFFFFFF00000000ull) | (uint32_t)(~(uint32_t)(i0 + v));
            const uint64_t bin = key[j] >> 52;
            if (ok[v] && (all || bin > d)) selm |= 1u << j;
            else if (ok[v] && bin == d) tiem |= 1u << j;
        }
    }
    // slots in the row's two lists: warp prefix sums, then one global atomic
    // per list for the whole CTA (the 32 or more CTAs of a row share the counters)
    const int ns = __popc(selm), nt = __popc(tiem);
    const int is = warp_incl_scan(ns), it = warp_incl_scan(nt);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __shared__ int wsel[TC_THREADS / 32], wtie[TC_THREADS / 32], cbase[2];
    if (lane == 31) {
        wsel[warp] = is;
        wtie[warp] = it;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int ts = 0, tt = 0;
        for (int w = 0; w < TC_THREADS / 32; w++) {
            const int a1 = wsel[w], a2 = wtie[w];
            wsel[w] = ts;
            wtie[w] = tt;
            ts += a1;
            tt += a2;
        }
        cbase[0] = ts ? atomicAdd(ws.cnt + 4 * r, ts) : 0;
        cbase[1] = tt ? atomicAdd(ws.cnt + 4 * r + 1, tt) : 0;
    }
    __syncthreads();
    int bs = cbase[0] + wsel[warp] + is - ns;
    int bt = cbase[1] + wtie[warp] + it - nt;
#pragma unroll
    for (int j = 0; j < TC_PER; j++) {
        if (selm & (1u << j)) {
            if (bs < a.k) ws.sel[r * a.k + bs] = (int32_t)(~(uint32_t)key[j]);
            bs++;
        } else if (tiem & (1u << j)) {
            if (bt < TK_BUF) ws.tie[r * TK_BUF + bt] = key[j];
            bt++;
        }
    }
}

// Block-wide exclusive prefix sum of v over the CTA's threads.
__device__ __forceinline__ int block_excl_scan(int v, TopkState &st) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int incl = warp_incl_scan(v);
    if (lane == 31) st.wsum[warp] = (uint32_t)incl;
    __syncthreads();
    int off = 0;
    for (int w = 0; w < warp; w++) off += (int)st.wsum[w];
    __syncthreads();
    return off + incl - v;
}

// Short tie lists are resolved by rank: the keys are distinct, so key i is
// among the best kk of the list iff fewer than kk keys of the list exceed it.
// Every thread of a warp reads the same list entry at a time (a broadcast);
// with at most RANK_MAX keys this is cheaper than further digit passes, each
// of which costs several block-wide barriers (1,024 keys measured 11 us slower
// per 1M step than the digit passes; the 4K step's short lists gain 2 us).
constexpr int RANK_MAX = 256;
template <int NT, typename F>
__device__ __forceinline__ void rank_select(const uint64_t *list, int n, int kk, F take) {
    for (int i = threadIdx.x; i < n; i += NT) {
        const uint64_t ki = list[i];
        int above = 0;
#pragma unroll 4
        for (int j = 0; j < n; j++) above += list[j] > ki ? 1 : 0;
        if (above < kk) take(ki);
    }
}

// Resolves the threshold bin's tie list (nbuf keys in sh.buf, all inside bin
// st.digit of the first 12-bit digit): the remaining digits run over the list
// and the tie keys at or above the k-th are appended to sh.sel as indices.
// st.above and st.match come from find_digit over the first-digit histogram.
__device__ void resolve_ties(TopkShared sh, TopkState &st, int nbuf, int k) {
    if (threadIdx.x == 0) {
        st.kk = k - (int)st.above;
        st.prefix = (uint64_t)st.digit << 52;
        st.mask = (uint64_t)(TK_HIST - 1) << 52;
    }
    __syncthreads();
    if (st.match != (uint32_t)st.kk && nbuf <= RANK_MAX) {
        rank_select<TK_THREADS>(sh.buf, nbuf, st.kk, [&](uint64_t key) {
            const int s2 = atomicAdd(&st.nsel, 1);
            if (s2 < TK_MAXK) sh.sel[s2] = (int32_t)(~(uint32_t)key);
        });
        return;
    }
    if (st.match != (uint32_t)st.kk) {
        // remaining digits: 10 + 10 bits finish the score, then the index bytes
        const int widths[6] = {10, 10, 8, 8, 8, 8};
        int shift = 52;
        for (int wi = 0; wi < 6; wi++) {
            shift -= widths[wi];
            const int NB = 1 << widths[wi];
            smem_hist_pass(sh.buf, nbuf, sh.hist, NB, shift, st.prefix, st.mask);
            find_digit(sh.hist, NB, st.kk, st);
            if (threadIdx.x == 0) {
                st.kk -= (int)st.above;
                st.prefix |= (uint64_t)st.digit << shift;
                st.mask |= (uint64_t)(NB - 1) << shift;
            }
            __syncthreads();
            if (st.match == (uint32_t)st.kk) break;
        }
    }
    const uint64_t p = st.prefix, m = st.mask;
    for (int i = threadIdx.x; i < nbuf; i += TK_THREADS) {
        const uint64_t key = sh.buf[i];
        if ((key & m) >= p) {
            const int s2 = atomicAdd(&st.nsel, 1);
            if (s2 < TK_MAXK) sh.sel[s2] = (int32_t)(~(uint32_t)key);
        }
    }
}

// Writes the selected candidate indices sh.sel[0..nsel) of row r in index
// order (their positions, or the indices themselves without cand_pos), then
// -1 up to k: a bitmap over [0, n) in sh.buf and a block prefix count of its
// set bits give every selected index its output slot.
__device__ void emit_in_index_order(const TopkArgs &a, int64_t r, TopkShared sh, TopkState &st,
                                    int nsel) {
    int32_t *out = a.out + r * a.k;
    uint32_t *bm = reinterpret_cast<uint32_t *>(sh.buf);
    const int nwords = (int)((a.n + 31) / 32);
    for (int i = threadIdx.x; i < nwords; i += TK_THREADS) bm[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < nsel; i += TK_THREADS) {
        const int idx = sh.sel[i];
        atomicOr(&bm[idx >> 5], 1u << (idx & 31));
    }
    __syncthreads();
    const int per = (nwords + TK_THREADS - 1) / TK_THREADS;
    const int w0 = threadIdx.x * per;
    int c = 0;
    for (int i = 0; i < per; i++)
        if (w0 + i < nwords) c += __popc(bm[w0 + i]);
    int rank = block_excl_scan(c, st);
    for (int i = 0; i < per; i++) {
        if (w0 + i >= nwords) break;
        uint32_t bits = bm[w0 + i];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            const int64_t idx = (int64_t)(w0 + i) * 32 + b;
            if (rank < a.k) out[rank] = a.cand_pos ? a.cand_pos[r * a.n + idx] : (int32_t)idx;
            rank++;
        }
    }
    for (int i = nsel + threadIdx.x; i < a.k; i += TK_THREADS) out[i] = -1;
}

__global__ void __launch_bounds__(TK_THREADS, 1) topk_finish_kernel(TopkArgs a, TopkHistWs ws) {
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ TopkState st;
    TopkShared sh = topk_shared(smem_raw);
    const int64_t r = blockIdx.x;
    const int nsel0 = min(ws.cnt[4 * r], a.k);
    const int ntie = ws.cnt[4 * r + 1];
    if (threadIdx.x == 0) {
        st.prefix = 0;
        st.mask = 0;
        st.nsel = 0;
        st.nbuf = 0;
    }
    hist_threshold<TK_THREADS>(ws.hist + r * TK_HIST, a.k, st);
    const bool all = st.total <= (uint32_t)a.k;
    if ((!all && ntie > TK_BUF) || a.n > TF_MAX_N) {
        __syncthreads();
        topk_row_full(a, r, sh, st);  // rare: the tie list or the bitmap does not fit
    } else {
        load_batched(sh.sel, ws.sel + r * a.k, nsel0);
        if (threadIdx.x == 0) st.nsel = nsel0;
        if (!all) {
            load_batched(sh.buf, ws.tie + r * TK_BUF, ntie);
            resolve_ties(sh, st, ntie, a.k);
        }
        __syncthreads();
        emit_in_index_order(a, r, sh, st, min(st.nsel, a.k));
    }
    // leave the histogram and counters of this row clear for the next producer
    __syncthreads();
    for (int b = threadIdx.x; b < TK_HIST; b += TK_THREADS) ws.hist[r * TK_HIST + b] = 0;
    if (threadIdx.x < 3) ws.cnt[4 * r + threadIdx.x] = 0;
}

// Rows of at most TS_MAX_N candidates skip the global lists: one CTA per row
// takes the threshold bin from the producer's histogram, reads its candidates
// once (16 per thread per pass, one shared atomic per warp per list), keeps
// the indices above the bin and the bin's keys in shared memory, resolves the
// ties and emits in index order. A tie list longer than its buffer falls back
// to the whole single-CTA selection. Clears the row's histogram.
constexpr int64_t TS_MAX_N = 65536;
constexpr int TS_PER = 16;

__device__ void topk_row_hist_body(const TopkArgs &a, int64_t r, uint32_t *ghist, TopkShared sh,
                                   TopkState &st) {
    const int lane = threadIdx.x & 31;
    int64_t nv = a.n;
    if (a.n_valid) {
        const int64_t v = a.n_valid[r];
        nv = v < 0 ? 0 : (v < a.n ? v : a.n);
    }
    if (a.cand_pos == nullptr && nv <= a.k) {
        // a row of at most k candidates: every index is selected, in order
        int32_t *out = a.out + r * a.k;
        for (int i = threadIdx.x; i < a.k; i += TK_THREADS) out[i] = i < nv ? i : -1;
        for (int b = threadIdx.x; b < TK_HIST; b += TK_THREADS) ghist[r * TK_HIST + b] = 0;
        if (threadIdx.x == 0) st.nsel = (int)nv;
        return;
    }
    if (threadIdx.x == 0) {
        st.prefix = 0;
        st.mask = 0;
        st.nsel = 0;
        st.nbuf = 0;
    }
    hist_threshold<TK_THREADS>(ghist + r * TK_HIST, a.k, st);
    const bool all = st.total <= (uint32_t)a.k;
    const uint32_t d = (uint32_t)st.digit;
    const bool vec = ((r * a.n) % 4 == 0) && aligned16(a.score) &&
                     (a.cand_pos == nullptr || aligned16(a.cand_pos));
    for (int64_t b0 = 0; b0 < nv; b0 += (int64_t)TK_THREADS * TS_PER) {
        uint32_t ob[TS_PER];  // order-preserving score bits
        uint32_t selm = 0, tiem = 0;
#pragma unroll
        for (int u = 0; u < TS_PER / 4; u++) {
            const int64_t i0 = b0 + 4 * ((int64_t)u * TK_THREADS + threadIdx.x);
            uint64_t pk[4];
            bool ok[4];
            load_cand4(a, r, i0, nv, vec, pk, ok);
#pragma unroll
            for (int v = 0; v < 4; v++) {
                const int j = 4 * u + v;
                ob[j] = (uint32_t)(pk[v] >> 32);
                const uint32_t bin = ob[j] >> 20;
                if (ok[v] && (all || bin > d)) selm |= 1u << j;
                else if (ok[v] && bin == d) tiem |= 1u << j;
            }
        }
        const int ns = __popc(selm), nt = __popc(tiem);
        const int is = warp_incl_scan(ns), it = warp_incl_scan(nt);
        int bs = 0, bt = 0;
        if (lane == 31) {
            if (is) bs = atomicAdd(&st.nsel, is);
            if (it) bt = atomicAdd(&st.nbuf, it);
        }
        bs = __shfl_sync(0xffffffffu, bs, 31) + is - ns;
        bt = __shfl_sync(0xffffffffu, bt, 31) + it - nt;
#pragma unroll
        for (int j = 0; j < TS_PER; j++) {
            const uint32_t i = (uint32_t)(b0 + 4 * ((j >> 2) * TK_THREADS + threadIdx.x) + (j & 3));
            if (selm & (1u << j)) {
                if (bs < TK_MAXK) sh.sel[bs] = (int32_t)i;
                bs++;
            } else if (tiem & (1u << j)) {
                if (bt < TK_BUF) sh.buf[bt] = ((uint64_t)ob[j] << 32) | (uint32_t)~i;
                bt++;
            }
        }
    }
    __syncthreads();
    if (!all && st.nbuf > TK_BUF) {
        __syncthreads();
        topk_row_full(a, r, sh, st);  // rare: the tie list does not fit
    } else {
        if (!all) resolve_ties(sh, st, st.nbuf, a.k);
        __syncthreads();
        emit_in_index_order(a, r, sh, st, min(st.nsel, a.k));
    }
    __syncthreads();
    for (int b = threadIdx.x; b < TK_HIST; b += TK_THREADS) ghist[r * TK_HIST + b] = 0;
}

__global__ void __launch_bounds__(TK_THREADS, 1) topk_row_hist_kernel(TopkArgs a, uint32_t *ghist) {
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ TopkState st;
    topk_row_hist_body(a, blockIdx.x, ghist, topk_shared(smem_raw), st);
}

// ------------------------------------------------------------------ short rows, fast path
// Rows of at most FT_N candidates (the 16,384 pooled tokens of a Reindex layer)
// with k <= FT_K and the producer's first-digit histogram: one CTA of FT_THREADS
// threads per row holds every candidate's position, and the rank keys (score
// order bits, inverted index) of the threshold bin's candidates, in shared
// memory.
//  1. The histogram row (4 bins per thread, in registers) gives the threshold
//     bin d by one block-wide suffix scan.
//  2. One pass over the candidates (16 per thread, 16-byte loads): positions
//     to shared memory; the candidates above d go straight to a bitmap over
//     the indices, the keys of bin d to a compact tie list.
//  3. When only part of bin d is taken, its best keys are found over the tie
//     list: by rank for a short list, else by the remaining digits (10, 10,
//     then the index bytes); every key is distinct, so the last digit decides.
//  4. Emission in index order (= position order inside the step) through a
//     block prefix count of the bitmap words; -1 padding; the histogram row is
//     cleared for the next producer.
constexpr int FT_THREADS = 1024;
constexpr int FT_N = 16384;
constexpr int FT_K = 512;
constexpr int FT_PER = FT_N / FT_THREADS;                       // 16 candidates per thread
constexpr int FT_BPT = TK_HIST / FT_THREADS;                    // 4 histogram bins per thread
static_assert(FT_BPT % 4 == 0 && FT_PER % 4 == 0 && FT_N / 32 <= FT_THREADS, "fast-path shape");
constexpr size_t FT_SMEM = (size_t)FT_N * 8 + (size_t)FT_N * 4 + (size_t)(FT_N / 32) * 4 + 1024 * 4;

__global__ void __launch_bounds__(FT_THREADS, 1) topk_fast_kernel(TopkArgs a, uint32_t *ghist) {
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ TopkState st;
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);
    int32_t *pos = reinterpret_cast<int32_t *>(smem_raw + (size_t)FT_N * 8);
    uint32_t *bm = reinterpret_cast<uint32_t *>(smem_raw + (size_t)FT_N * 12);
    uint32_t *hist = bm + FT_N / 32;  // 1024 bins for the refinement digits
    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int nv = (int)a.n;
    if (a.n_valid) {
        const int64_t v = a.n_valid[r];
        nv = v < 0 ? 0 : (v < a.n ? (int)v : (int)a.n);
    }
    const int k = a.k;
    // ---- 1. threshold bin from the histogram row (bins [FT_BPT tid, FT_BPT tid + FT_BPT))
    uint32_t hb[FT_BPT];
    {
        const uint4 *hp = reinterpret_cast<const uint4 *>(ghist + r * TK_HIST) + (FT_BPT / 4) * tid;
#pragma unroll
        for (int q = 0; q < FT_BPT / 4; q++) {
            const uint4 h = hp[q];
            hb[4 * q] = h.x;
            hb[4 * q + 1] = h.y;
            hb[4 * q + 2] = h.z;
            hb[4 * q + 3] = h.w;
        }
    }
    for (int i = tid; i < FT_N / 32; i += FT_THREADS) bm[i] = 0;
    uint32_t local = 0;
#pragma unroll
    for (int j = 0; j < FT_BPT; j++) local += hb[j];
    uint32_t x = local;  // inclusive suffix sum over the lanes of the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
    }
    if (lane == 0) st.wsum[warp] = x;
    if (tid == 0) {
        st.digit = -1;
        st.nbuf = 0;
    }
    __syncthreads();
    uint32_t above = x - local, total = 0;
    for (int w = 0; w < FT_THREADS / 32; w++) {
        total += st.wsum[w];
        if (w > warp) above += st.wsum[w];
    }
    const bool all = total <= (uint32_t)k;
#pragma unroll
    for (int j = FT_BPT - 1; j >= 0; j--) {
        if (!all && above < (uint32_t)k && above + hb[j] >= (uint32_t)k) {
            st.digit = FT_BPT * tid + j;
            st.above = above;
            st.match = hb[j];
        }
        above += hb[j];
    }
    __syncthreads();
    const int d = all ? -1 : st.digit;
    // ---- 2. candidates (16 per thread, 16-byte loads): the positions to shared
    // memory, the candidates above d to the bitmap and the threshold bin's keys
    // to a compact tie list (rank key with the index, not the position, in the
    // low bits: ties go to the lower index, which inside the step is the lower
    // position)
    const bool vec = ((r * a.n) % 4 == 0) && aligned16(a.score) &&
                     (a.cand_pos == nullptr || aligned16(a.cand_pos));
#pragma unroll
    for (int u = 0; u < FT_PER / 4; u++) {
        const int i0 = 4 * (u * FT_THREADS + tid);
        uint64_t kq[4];
        bool ok[4];
        load_cand4(a, r, i0, nv, vec, kq, ok);
#pragma unroll
        for (int v = 0; v < 4; v++) {
            const int i = i0 + v;
            pos[i] = ok[v] ? rank_key_pos(kq[v]) : -1;
            const int bin = (int)(kq[v] >> 52);
            if (ok[v] && (all || bin > d)) atomicOr(&bm[i >> 5], 1u << (i & 31));
            else if (ok[v] && bin == d)
                keys[atomicAdd(&st.nbuf, 1)] = (kq[v] & 0xFFFFFFFF00000000ull) | (uint32_t)~(uint32_t)i;
        }
    }
    if (tid == 0) {
        st.kk = all ? 0 : k - (int)st.above;
        st.prefix = (uint64_t)(all ? 0 : d) << 52;
        st.mask = (uint64_t)(TK_HIST - 1) << 52;
    }
    __syncthreads();
    // ---- 3. the threshold bin (its keys in the tie list): all of it, or its
    // best kk by the remaining digits
    if (!all && st.nbuf != st.kk && st.nbuf <= RANK_MAX) {
        rank_select<FT_THREADS>(keys, st.nbuf, st.kk, [&](uint64_t key) {
            const int idx = (int)~(uint32_t)key;
            atomicOr(&bm[idx >> 5], 1u << (idx & 31));
        });
        __syncthreads();
    } else if (!all) {
        const int ntie = st.nbuf;
        if (ntie != st.kk) {
            const int widths[6] = {10, 10, 8, 8, 8, 8};
            int shift = 52;
            for (int wi = 0; wi < 6; wi++) {
                shift -= widths[wi];
                const int NB = 1 << widths[wi];
                smem_hist_pass<FT_THREADS>(keys, ntie, hist, NB, shift, st.prefix, st.mask);
                find_digit<FT_THREADS>(hist, NB, st.kk, st);
                if (tid == 0) {
                    st.kk -= (int)st.above;
                    st.prefix |= (uint64_t)st.digit << shift;
                    st.mask |= (uint64_t)(NB - 1) << shift;
                }
                __syncthreads();
                if (st.match == (uint32_t)st.kk) break;
            }
        }
        const uint64_t p = st.prefix, m = st.mask;
        for (int i = tid; i < ntie; i += FT_THREADS) {
            const uint64_t key = keys[i];
            if ((key & m) >= p) {
                const int idx = (int)~(uint32_t)key;
                atomicOr(&bm[idx >> 5], 1u << (idx & 31));
            }
        }
        __syncthreads();
    }
    // ---- 4. emission in index order: thread t owns bitmap word t
    const uint32_t word = tid < FT_N / 32 ? bm[tid] : 0u;
    const int c = __popc(word);
    int rank = block_excl_scan(c, st);
    int32_t *out = a.out + r * a.k;
    uint32_t bits = word;
    while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (rank < k) out[rank] = pos[32 * tid + b];
        rank++;
    }
    if (tid == FT_THREADS - 1) st.nsel = rank;
    // clear the histogram row for the next producer
    {
        uint4 *hp = reinterpret_cast<uint4 *>(ghist + r * TK_HIST) + (FT_BPT / 4) * tid;
#pragma unroll
        for (int q = 0; q < FT_BPT / 4; q++) hp[q] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    for (int i = st.nsel + tid; i < k; i += FT_THREADS) out[i] = -1;
}

// ------------------------------------------------------------------ pool + tokens
// The decode Full layer's selection after its scan, in one CTA per row: the
// pool (best P blocks, from the producer's histogram, as the two selection
// kernels above do) and then the row's top-K tokens among the pooled blocks'
// tokens. The pooled tokens' rank keys are gathered into shared memory in pool
// order, which is position order (the pool is written ascending), and selected
// there: a 12-bit first digit, then the remaining digits of the threshold
// bin's keys, then emission in index order (= ascending positions) through a
// bitmap. An empty slot holds key 0, which no finite score produces.
constexpr int PT_MAX = kPoolBlocks * kBlockTokens;                  // 16,384 pooled tokens
// Rows of up to this many blocks take the one-kernel path (one CTA reads the
// row); longer rows are compacted by many CTAs first. Taking the 1M rows
// (131,072 blocks) in one CTA as well measured 1.683 against 1.670 ms per step
// (same B200).
constexpr int64_t PT_ONE_CTA_MAX_N = TS_MAX_N;
constexpr size_t PT_SMEM = TK_HIST * 4 + TK_MAXK * 4 + (size_t)PT_MAX * 8;  // 160 KB
static_assert((size_t)PT_MAX * 8 >= (size_t)TK_BUF * 8, "the key array holds the tie buffer");

__device__ __forceinline__ TopkShared pool_tokens_shared(uint8_t *smem_raw) {
    return TopkShared{reinterpret_cast<uint32_t *>(smem_raw),
                      reinterpret_cast<uint64_t *>(smem_raw + TK_HIST * 4 + TK_MAXK * 4),
                      reinterpret_cast<int32_t *>(smem_raw + TK_HIST * 4)};
}

struct PoolTokArgs {
    const float *tok;        // [R][cap] token scores of the scan
    const int64_t *ctx_len;  // [R] visible length of each row
    int64_t cap;
    int k;                   // tokens to keep (<= TK_MAXK)
    int32_t *top;            // [R][k] ascending positions, -1 padded
};

// Top-pa.k tokens of row r among the tokens of the a.k pool blocks this CTA
// just wrote to a.out (row r, ascending block ids, -1 padded). All threads of
// the CTA, after a barrier that follows the pool's writes.
// identity_n >= 0: the pool is blocks 0 .. identity_n - 1 (a row of at most P
// blocks), so it is not read back. dblk >= 0: the first-digit bin of the
// row's pa.k-th best block score. The best pa.k tokens lie in the best pa.k
// blocks (every block ranked ahead of a token's block holds a token ranked
// ahead of that token), so only the pooled blocks whose score reaches bin dblk
// are candidates: a superset of those blocks, usually about a quarter of the
// pool.
__device__ void pool_tokens_select(const TopkArgs &a, const PoolTokArgs &pa, int64_t r,
                                   TopkShared sh, TopkState &st, int identity_n, int dblk) {
    const int P = a.k;
    uint64_t *keys = sh.buf;
    int64_t V = pa.ctx_len[r];
    if (V > pa.cap) V = pa.cap;
    const int32_t *pool = a.out + r * (int64_t)P;
    // the pool is ascending and -1 padded: only its valid entries' tokens are
    // candidates (a row shorter than the pool has fewer)
    int npool = 0;
    if (identity_n >= 0) {
        npool = identity_n < P ? identity_n : P;
    } else {
        for (int i0 = 0; i0 < P; i0 += TK_THREADS)
            npool += __syncthreads_count(i0 + (int)threadIdx.x < P && pool[i0 + threadIdx.x] >= 0);
    }
    // candidate blocks in pool order (ascending), in the histogram's space until
    // their tokens are gathered
    int32_t *cand = reinterpret_cast<int32_t *>(sh.hist);
    const bool filtered = identity_n < 0 && dblk >= 0;
    if (filtered) {
        constexpr int PPT_MAX = (kPoolBlocks + TK_THREADS - 1) / TK_THREADS;
        const int ppt = (P + TK_THREADS - 1) / TK_THREADS;  // <= PPT_MAX (P <= kPoolBlocks)
        int32_t cb[PPT_MAX];
        int c = 0;
#pragma unroll
        for (int j = 0; j < PPT_MAX; j++) {
            const int sl = ppt * (int)threadIdx.x + j;
            const int32_t blk = (j < ppt && sl < npool) ? pool[sl] : -1;
            cb[j] = (blk >= 0 && (int)hist_bin(a.score[r * a.n + blk]) >= dblk) ? blk : -1;
            c += cb[j] >= 0;
        }
        int off = block_excl_scan(c, st);
#pragma unroll
        for (int j = 0; j < PPT_MAX; j++)
            if (cb[j] >= 0) cand[off++] = cb[j];
        if (threadIdx.x == TK_THREADS - 1) st.nsel = off;
        __syncthreads();
        npool = st.nsel;
    }
    const int n = npool * kBlockTokens;
    const float *tok = pa.tok + r * pa.cap;
    for (int i = threadIdx.x; i < n; i += TK_THREADS) {
        const int32_t blk = filtered ? cand[i >> 3] : identity_n >= 0 ? (i >> 3) : pool[i >> 3];
        const int64_t pos = 8 * (int64_t)blk + (i & 7);
        keys[i] = (blk >= 0 && pos < V) ? rank_key(tok[pos], (int32_t)pos) : 0ull;
    }
    if (filtered) __syncthreads();  // the candidate list is read; the histogram takes its space
    for (int b = threadIdx.x; b < TK_HIST; b += TK_THREADS) sh.hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += TK_THREADS) {
        const uint64_t key = keys[i];
        if (key) atomicAdd(&sh.hist[key >> 52], 1u);
    }
    __syncthreads();
    find_digit(sh.hist, TK_HIST, pa.k, st);
    const bool all = st.total <= (uint32_t)pa.k;
    const uint64_t d = (uint64_t)st.digit;
    if (threadIdx.x == 0) {
        st.kk = pa.k - (int)st.above;
        st.prefix = d << 52;
        st.mask = (uint64_t)(TK_HIST - 1) << 52;
    }
    __syncthreads();
    // The threshold bin's keys are resolved over a compact list in the sel
    // region when they fit there (with the index, which orders like the
    // position, in their low bits), else over the whole key array.
    uint64_t *ties = reinterpret_cast<uint64_t *>(sh.sel);
    const bool partial = !all && st.match != (uint32_t)st.kk;
    const bool listed = partial && st.match <= (uint32_t)(TK_MAXK / 2);
    if (listed) {
        if (threadIdx.x == 0) st.nbuf = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += TK_THREADS) {
            const uint64_t key = keys[i];
            if (key && (key >> 52) == d)
                ties[atomicAdd(&st.nbuf, 1)] = (key & 0xFFFFFFFF00000000ull) | (uint32_t)~(uint32_t)i;
        }
        __syncthreads();
    }
    const bool ranked = listed && st.nbuf <= RANK_MAX;
    if (partial && !ranked) {
        // only part of the threshold bin is taken: further digits over its keys
        const uint64_t *tk = listed ? ties : keys;
        const int ntk = listed ? st.nbuf : n;
        const int widths[6] = {10, 10, 8, 8, 8, 8};
        int shift = 52;
        for (int wi = 0; wi < 6; wi++) {
            shift -= widths[wi];
            const int NB = 1 << widths[wi];
            smem_hist_pass(tk, ntk, sh.hist, NB, shift, st.prefix, st.mask);
            find_digit(sh.hist, NB, st.kk, st);
            if (threadIdx.x == 0) {
                st.kk -= (int)st.above;
                st.prefix |= (uint64_t)st.digit << shift;
                st.mask |= (uint64_t)(NB - 1) << shift;
            }
            __syncthreads();
            if (st.match == (uint32_t)st.kk) break;
        }
    }
    const uint64_t p = st.prefix, m = st.mask;
    // bitmap of the selected indices over [0, n), in the histogram's space
    // a warp covers 32 consecutive keys, one bitmap word: one ballot writes it
    uint32_t *bm = sh.hist;
    const int nwords = (n + 31) / 32;
    for (int i0 = 0; i0 < nwords * 32; i0 += TK_THREADS) {
        const int i = i0 + (int)threadIdx.x;
        bool take = false;
        if (i < n) {
            const uint64_t key = keys[i];
            take = key && (all || (key >> 52) > d || (!listed && (key & m) >= p && (key >> 52) == d));
        }
        const uint32_t word = __ballot_sync(0xffffffffu, take);
        if ((threadIdx.x & 31) == 0 && i < nwords * 32) bm[i >> 5] = word;
    }
    if (ranked) {
        __syncthreads();  // the tie bits go on top of the words written above
        rank_select<TK_THREADS>(ties, st.nbuf, st.kk, [&](uint64_t key) {
            const int idx = (int)~(uint32_t)key;
            atomicOr(&bm[idx >> 5], 1u << (idx & 31));
        });
    } else if (listed) {
        __syncthreads();  // the tie bits go on top of the words written above
        for (int i = threadIdx.x; i < st.nbuf; i += TK_THREADS) {
            const uint64_t key = ties[i];
            if ((key & m) >= p) {
                const int idx = (int)~(uint32_t)key;
                atomicOr(&bm[idx >> 5], 1u << (idx & 31));
            }
        }
    }
    __syncthreads();
    const int per = (nwords + TK_THREADS - 1) / TK_THREADS;
    const int w0 = threadIdx.x * per;
    int c = 0;
    for (int i = 0; i < per; i++)
        if (w0 + i < nwords) c += __popc(bm[w0 + i]);
    int rank = block_excl_scan(c, st);
    int32_t *out = pa.top + r * (int64_t)pa.k;
    for (int i = 0; i < per; i++) {
        if (w0 + i >= nwords) break;
        uint32_t bits = bm[w0 + i];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            if (rank < pa.k) out[rank] = rank_key_pos(keys[(w0 + i) * 32 + b]);
            rank++;
        }
    }
    // the last thread's rank is the number selected: -1 after them
    if (threadIdx.x == TK_THREADS - 1) st.nsel = rank;
    __syncthreads();
    for (int i = st.nsel + threadIdx.x; i < pa.k; i += TK_THREADS) out[i] = -1;
}

// Pool of row r from the compacted global lists (as topk_finish_kernel), then
// the row's top tokens among the pooled tokens. All threads of a CTA of
// TK_THREADS; the lists and counters of the row are complete and visible.
__device__ void finish_pool_tokens_row(const TopkArgs &a, const TopkHistWs &ws, const PoolTokArgs &pa,
                                       int64_t r, TopkShared sh, TopkState &st, int &dblk_s) {
    const int nsel0 = min(ws.cnt[4 * r], a.k);
    const int ntie = ws.cnt[4 * r + 1];
    if (threadIdx.x == 0) {
        st.prefix = 0;
        st.mask = 0;
        st.nsel = 0;
        st.nbuf = 0;
    }
    // the pool's threshold bin, and the bin of the pa.k-th best block score for
    // the token candidates, from one read of the histogram
    hist_threshold2<TK_THREADS>(ws.hist + r * TK_HIST, a.k, pa.k, st, &dblk_s);
    const bool all = st.total <= (uint32_t)a.k;
    if ((!all && ntie > TK_BUF) || a.n > TF_MAX_N) {
        __syncthreads();
        topk_row_full(a, r, sh, st);  // rare: the tie list or the bitmap does not fit
    } else {
        load_batched(sh.sel, ws.sel + r * a.k, nsel0);
        if (threadIdx.x == 0) st.nsel = nsel0;
        if (!all) {
            load_batched(sh.buf, ws.tie + r * TK_BUF, ntie);
            resolve_ties(sh, st, ntie, a.k);
        }
        __syncthreads();
        emit_in_index_order(a, r, sh, st, min(st.nsel, a.k));
    }
    // leave the histogram and counters of this row clear for the next producer
    __syncthreads();
    for (int b = threadIdx.x; b < TK_HIST; b += TK_THREADS) ws.hist[r * TK_HIST + b] = 0;
    if (threadIdx.x < 3) ws.cnt[4 * r + threadIdx.x] = 0;
    __syncthreads();
    pool_tokens_select(a, pa, r, sh, st, -1, dblk_s);
}

// Rows longer than PT_ONE_CTA_MAX_N blocks in one launch: CTA (x, r) compacts
// blocks [x TK_THREADS 4, ...) of row r into the row's global lists (the
// indices above the threshold bin and the bin's keys, slots by one global
// atomic per list per CTA), then takes a ticket; the last CTA of the row
// finishes the pool and selects the row's top tokens. The ticket is a release /
// acquire pair (fences around the atomic), so no CTA waits on another.
constexpr int TC2_SLICE = TK_THREADS * 4;  // candidates per CTA, one 16-byte load per thread

__global__ void __launch_bounds__(TK_THREADS, 1)
    topk_compact_pool_tokens_kernel(TopkArgs a, TopkHistWs ws, PoolTokArgs pa) {
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ TopkState st;
    __shared__ int dblk_s, last_s, wsel[TK_THREADS / 32], wtie[TK_THREADS / 32], cbase[2];
    const int64_t r = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t nv = a.n;
    if (a.n_valid) {
        const int64_t v = a.n_valid[r];
        nv = v < 0 ? 0 : (v < a.n ? v : a.n);
    }
    const int64_t i_beg = (int64_t)blockIdx.x * TC2_SLICE;
    if (i_beg < nv) {  // uniform over the CTA
        hist_threshold<TK_THREADS>(ws.hist + r * TK_HIST, a.k, st);
        const bool all = st.total <= (uint32_t)a.k;
        const uint64_t d = (uint64_t)st.digit;
        const bool vec = ((r * a.n) % 4 == 0) && aligned16(a.score) &&
                         (a.cand_pos == nullptr || aligned16(a.cand_pos));
        const int64_t i0 = i_beg + 4 * (int64_t)threadIdx.x;
        uint64_t pk[4];
        bool ok[4];
        load_cand4(a, r, i0, nv, vec, pk, ok);
        uint32_t selm = 0, tiem = 0;
#pragma unroll
        for (int v = 0; v < 4; v++) {
            const uint64_t bin = pk[v] >> 52;
            if (ok[v] && (all || bin > d)) selm |= 1u << v;
            else if (ok[v] && bin == d) tiem |= 1u << v;
        }
        const int ns = __popc(selm), nt = __popc(tiem);
        const int is = warp_incl_scan(ns), it = warp_incl_scan(nt);
        if (lane == 31) {
            wsel[warp] = is;
            wtie[warp] = it;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int ts = 0, tt = 0;
            for (int w = 0; w < TK_THREADS / 32; w++) {
                const int a1 = wsel[w], a2 = wtie[w];
                wsel[w] = ts;
                wtie[w] = tt;
                ts += a1;
                tt += a2;
            }
            cbase[0] = ts ? atomicAdd(ws.cnt + 4 * r, ts) : 0;
            cbase[1] = tt ? atomicAdd(ws.cnt + 4 * r + 1, tt) : 0;
        }
        __syncthreads();
        int bs = cbase[0] + wsel[warp] + is - ns;
        int bt = cbase[1] + wtie[warp] + it - nt;
#pragma unroll
        for (int v = 0; v < 4; v++) {
            if (selm & (1u << v)) {
                if (bs < a.k) ws.sel[r * a.k + bs] = (int32_t)(i0 + v);
                bs++;
            } else if (tiem & (1u << v)) {
                // index-keyed: the ordered score bits above the inverted index
                if (bt < TK_BUF)
                    ws.tie[r * TK_BUF + bt] = (pk[v] & 0xFFFFFFFF00000000ull) | (uint32_t)~(uint32_t)(i0 + v);
                bt++;
            }
        }
    }
    // this CTA's list entries are written: take the row's ticket
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last_s = atomicAdd(ws.cnt + 4 * r + 2, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!last_s) return;
    __threadfence();  // every other CTA's entries of this row are visible
    finish_pool_tokens_row(a, ws, pa, r, pool_tokens_shared(smem_raw), st, dblk_s);
}

// Pool from one pass over the row (as topk_row_hist_kernel), then the row's top
// tokens among the pooled tokens.
__global__ void __launch_bounds__(TK_THREADS, 1)
    topk_row_pool_tokens_kernel(TopkArgs a, uint32_t *ghist, PoolTokArgs pa) {
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ TopkState st;
    __shared__ int dblk_s;
    TopkShared sh = pool_tokens_shared(smem_raw);
    // the bin of the pa.k-th best block score, for the token candidates
    hist_threshold<TK_THREADS>(ghist + blockIdx.x * TK_HIST, pa.k, st);
    if (threadIdx.x == 0) dblk_s = st.total <= (uint32_t)pa.k ? -1 : st.digit;
    topk_row_hist_body(a, blockIdx.x, ghist, sh, st);
    __syncthreads();
    // a row of at most P blocks pooled all of them, in order
    int64_t nv = a.n;
    if (a.n_valid) {
        const int64_t v = a.n_valid[blockIdx.x];
        nv = v < 0 ? 0 : (v < a.n ? v : a.n);
    }
    pool_tokens_select(a, pa, blockIdx.x, sh, st, nv <= a.k ? (int)nv : -1, dblk_s);
}

}  // namespace csa2

using namespace csa2;

namespace csa2 {

size_t topk_hist_ws_bytes(int R, int k) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    return topk_hist_zero_bytes(R) + up((size_t)R * k * 4) + up((size_t)R * TK_BUF * 8);
}

// The leading bytes of a selection workspace that must be zero before a
// producer fills it: the histogram rows and the counters.
size_t topk_hist_zero_bytes(int R) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    return up((size_t)R * TK_HIST * 4) + up((size_t)R * 4 * 4);
}

static TopkHistWs topk_hist_ws(void *base, int R, int k) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    char *p = static_cast<char *>(base);
    TopkHistWs w;
    w.hist = reinterpret_cast<uint32_t *>(p);
    p += up((size_t)R * TK_HIST * 4);
    w.cnt = reinterpret_cast<int *>(p);
    p += up((size_t)R * 4 * 4);
    w.sel = reinterpret_cast<int32_t *>(p);
    p += up((size_t)R * k * 4);
    w.tie = reinterpret_cast<uint64_t *>(p);
    return w;
}


// Selection of rows whose histogram (hist[r][4096], counters zero) the score
// producer has filled: one CTA per row for short rows, else compaction over
// many CTAs, then one finishing CTA per row.
int launch_topk_from_hist(const float *score, const int32_t *cand_pos, const int32_t *n_valid,
                          int R, int64_t n, int k, int32_t *out, void *ws, cudaStream_t s) {
    if (R == 0) return CSA2_OK;
    if (R > 65535) return CSA2_ERR_SHAPE;
    static PerDevice smem_set[3];
    if (!set_smem_limit_once(smem_set[0], topk_kernel, TK_SMEM) ||
        !set_smem_limit_once(smem_set[1], topk_finish_kernel, TK_SMEM) ||
        !set_smem_limit_once(smem_set[2], topk_row_hist_kernel, TK_SMEM))
        return CSA2_ERR_CUDA;
    TopkArgs a{score, cand_pos, n_valid, R, n, k, out};
    TopkHistWs w = topk_hist_ws(ws, R, k);
    if (n <= FT_N && k <= FT_K) {
        static PerDevice fast_set;
        if (!set_smem_limit_once(fast_set, topk_fast_kernel, FT_SMEM)) return CSA2_ERR_CUDA;
        return launch_kernel(true, topk_fast_kernel, dim3(R), dim3(FT_THREADS), FT_SMEM, s, a, w.hist);
    }
    if (n <= TS_MAX_N)
        return launch_kernel(true, topk_row_hist_kernel, dim3(R), dim3(TK_THREADS), TK_SMEM, s, a,
                             w.hist);
    const int64_t slices = (n + TC_SLICE - 1) / TC_SLICE;
    const int st = launch_kernel(true, topk_compact_kernel, dim3((unsigned)slices, (unsigned)R),
                                 dim3(TC_THREADS), 0, s, a, w);
    if (st) return st;
    return launch_kernel(true, topk_finish_kernel, dim3(R), dim3(TK_THREADS), TK_SMEM, s, a, w);
}

// The decode Full layer's pool (k = P blocks of the block scores blk, whose
// histogram the scan filled) and the top ktop tokens among the pooled tokens
// (token scores tok [R][cap]): written to pool and top. One CTA per row, or for
// rows longer than PT_ONE_CTA_MAX_N blocks a compaction over many CTAs per row
// whose last CTA finishes the row: one launch either way.
int launch_pool_and_tokens(const float *blk, const int32_t *n_blk, int R, int64_t nblk, int P,
                           int32_t *pool, void *ws, const float *tok, const int64_t *ctx_len,
                           int64_t cap, int ktop, int32_t *top, cudaStream_t s) {
    if (R == 0) return CSA2_OK;
    if (R > 65535 || P * kBlockTokens > PT_MAX || ktop > TK_MAXK) return CSA2_ERR_SHAPE;
    static PerDevice smem_set[2];
    if (!set_smem_limit_once(smem_set[0], topk_compact_pool_tokens_kernel, PT_SMEM) ||
        !set_smem_limit_once(smem_set[1], topk_row_pool_tokens_kernel, PT_SMEM))
        return CSA2_ERR_CUDA;
    TopkArgs a{blk, nullptr, n_blk, R, nblk, P, pool};
    PoolTokArgs pa{tok, ctx_len, cap, ktop, top};
    TopkHistWs w = topk_hist_ws(ws, R, P);
    if (nblk <= PT_ONE_CTA_MAX_N)
        return launch_kernel(true, topk_row_pool_tokens_kernel, dim3(R), dim3(TK_THREADS), PT_SMEM, s,
                             a, w.hist, pa);
    const int64_t slices = (nblk + TC2_SLICE - 1) / TC2_SLICE;
    if (slices > 65535) return CSA2_ERR_SHAPE;
    return launch_kernel(true, topk_compact_pool_tokens_kernel, dim3((unsigned)slices, (unsigned)R),
                         dim3(TK_THREADS), PT_SMEM, s, a, w, pa);
}

}  // namespace csa2

extern "C" size_t csa2_topk_workspace_size(int R, int64_t n, int k) {
    (void)R;
    (void)n;
    (void)k;
    return 0;
}

extern "C" int csa2_topk(const float *score, const int32_t *cand_pos, const int32_t *n_valid, int R,
                         int64_t n, int k, int32_t *out, void *ws, size_t ws_bytes, void *stream) {
    (void)ws;
    (void)ws_bytes;
    if (!score || !out) return CSA2_ERR_NULL;
    if (R < 0 || n < 1 || n >= ((int64_t)1 << 31) || k < 1 || k > TK_MAXK) return CSA2_ERR_SHAPE;
    if (R == 0) return CSA2_OK;
    static PerDevice smem_set;
    if (!set_smem_limit_once(smem_set, topk_kernel, TK_SMEM)) return CSA2_ERR_CUDA;
    TopkArgs a{score, cand_pos, n_valid, R, n, k, out};
    topk_kernel<<<R, TK_THREADS, TK_SMEM, (cudaStream_t)stream>>>(a);
    return launch_status();
}
