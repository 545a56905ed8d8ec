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

// Block-wide: given hist[0..NB), find the bin d where the count of keys at or
// above it first reaches kk (scanning from the top bin down).
__device__ void find_digit(const uint32_t *hist, int NB, int kk, TopkState &st) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int BPT = (NB + TK_THREADS - 1) / TK_THREADS;
    const int b0 = tid * BPT;
    uint32_t local = 0;
    for (int j = 0; j < BPT; j++)
        if (b0 + j < NB) local += hist[b0 + j];
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
    for (int w = 0; w < TK_THREADS / 32; w++) {
        all += st.wsum[w];
        if (w > warp) warps_above += st.wsum[w];
    }
    uint32_t above = (x - local) + warps_above;  // keys in bins above my bins
    for (int j = BPT - 1; j >= 0; j--) {
        const int bin = b0 + j;
        if (bin >= NB) continue;
        const uint32_t h = hist[bin];
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

__device__ void smem_hist_pass(const uint64_t *buf, int nbuf, uint32_t *hist, int NB, int shift,
                               uint64_t prefix, uint64_t mask) {
    for (int b = threadIdx.x; b < NB; b += TK_THREADS) hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < nbuf; i += TK_THREADS) {
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

__global__ void __launch_bounds__(TK_THREADS, 1) topk_kernel(TopkArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ TopkState st;
    TopkShared sh{reinterpret_cast<uint32_t *>(smem_raw),
                  reinterpret_cast<uint64_t *>(smem_raw + TK_HIST * 4),
                  reinterpret_cast<int32_t *>(smem_raw + TK_HIST * 4 + TK_BUF * 8)};
    const int64_t r = blockIdx.x;
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

}  // namespace csa2

using namespace csa2;

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
    static bool attr_set = false;
    if (!attr_set) {
        if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)TK_SMEM) != cudaSuccess)
            return CSA2_ERR_CUDA;
        attr_set = true;
    }
    TopkArgs a{score, cand_pos, n_valid, R, n, k, out};
    topk_kernel<<<R, TK_THREADS, TK_SMEM, (cudaStream_t)stream>>>(a);
    return launch_status();
}
