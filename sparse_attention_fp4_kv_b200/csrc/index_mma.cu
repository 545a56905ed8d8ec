// Multi-query indexer scan on tensor cores (chunked prefill; several queries
// per sequence).
//
// "DeepSeek-V4.1-Flash: 890 Bytes Per Token, 437x Smaller KV Cache", CSA2
// section: a Full layer scores the context with its indexer and builds the
// pool of up to 2,048 blocks of 8 tokens. With many queries per sequence (a
// prefill chunk) the scores form a dense int8 contraction
//     S[i][t] = sum_{h,d} q[i][h][d] * k[t][h][d]
// that belongs on the tensor cores: tcgen05.mma kind::i8 with exact int32
// accumulation, so the results are bit-identical to the dp4a scan.
//
// Persistent, warp-specialised CTA (192 threads, one per SM):
//   warp 0      TMA producer: 128-byte-swizzled tiles of Q (128 queries x 128 B)
//               and K (256 keys x 128 B) into a 4-stage shared-memory ring;
//   warp 1      TMEM owner and MMA issuer: 4 MMAs (M = 128, N = 256, K = 32)
//               per stage into one of two 256-column int32 accumulators;
//   warps 2-5   epilogue: one query row per thread, 32 key columns at a time
//               (the next TMEM load in flight while the current chunk is
//               stored); int32 -> fp32 (RNE) times the key scale (staged once
//               per tile in shared memory), causal mask (t <= query position),
//               8-token block maxima as 16-byte stores, token scores
//               transposed through shared memory so that every warp store
//               writes whole 128-byte row segments.
// Tiles are ordered query-tile fastest, so the CTAs working at the same time
// share key tiles in L2 and every key tile is read from HBM about once.
// All mbarrier waits are bounded; on timeout the kernel records an error flag
// and leaves its loops.
#include "tma.cuh"

namespace csa2 {
namespace imma {

constexpr int BM = 128;  // queries per tile
constexpr int BN = 256;  // keys per tile
constexpr int BK = 128;  // bytes of the indexer row per stage
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK;
constexpr int B_STAGE = BN * BK;
constexpr int THREADS = 192;
constexpr int BAR_BYTES = 256;
// per epilogue warp: a [32 rows][36] fp32 transpose tile (rows padded by 16 B so
// that both its row-wise and column-wise 16-byte accesses are conflict-free)
// and the tile's 256 key scales
constexpr int STG_LD = 36;
constexpr int EPI_WARP = 32 * STG_LD * 4 + BN * 4;
constexpr int EPI_OFF = STAGES * (A_STAGE + B_STAGE) + BAR_BYTES;
constexpr int SMEM_BYTES = EPI_OFF + 4 * EPI_WARP + 1024;
constexpr long WAIT_LIMIT = 1L << 26;

__device__ int g_imma_error = 0;

struct Args {
    const float *kscale;
    const int64_t *ctx_len;
    const int64_t *q_pos;
    int B, Nq, HD;
    int64_t cap, nblk_cap;
    float *tok;
    float *blk;
    int32_t *n_blk;
    int m_tiles, n_tiles;
    int64_t tiles;
    bool vec;      // token rows and key scales are 16-byte aligned
    bool vec_blk;  // block-score rows are 16-byte aligned
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (long it = 0; it < WAIT_LIMIT; it++) {
        uint32_t done;
        asm volatile(
            "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            "selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    atomicExch(&g_imma_error, 1);
    return false;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ uint64_t sdesc(uint32_t addr) {
    // 128-byte swizzle, K-major: 8-row atoms of 1024 B (SBO), LBO unused (16 B).
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)64 << 32) |
           (1ull << 46) | (2ull << 61);
}
// kind::i8 instruction descriptor: s32 accumulate, signed int8 A and B, K-major.
constexpr uint32_t IDESC = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);
__device__ __forceinline__ void mma_i8(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}" ::"r"(d),
        "l"(a), "l"(b), "r"(IDESC), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}
// 32 consecutive columns of this warp's 32 TMEM lanes; the registers are valid
// after tmem_ld_wait(v), which names them so that no use moves above the wait.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, int (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
        "%30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
          "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
          "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait(int (&v)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                   "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                   "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]), "+r"(v[17]),
                   "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]),
                   "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]),
                   "+r"(v[30]), "+r"(v[31])
                 :
                 : "memory");
}

struct Tile {
    int b, m0, n0;
};
__device__ __forceinline__ Tile tile_of(const Args &a, int64_t t) {
    Tile r;
    const int mt = (int)(t % a.m_tiles);
    const int64_t rest = t / a.m_tiles;
    r.n0 = (int)(rest % a.n_tiles) * BN;
    r.b = (int)(rest / a.n_tiles);
    r.m0 = mt * BM;
    return r;
}

__global__ void __launch_bounds__(THREADS, 1)
    index_mma_kernel(const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k, Args a) {
    grid_dep_wait();
    grid_dep_launch();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sm = smem_raw + (base - raw);
    const uint32_t a_s = base, b_s = base + STAGES * A_STAGE;
    const uint32_t bars = base + STAGES * (A_STAGE + B_STAGE);
    const uint32_t full = bars, empty = bars + 8 * STAGES;
    const uint32_t tfull = bars + 16 * STAGES, tempty = tfull + 16;
    uint32_t *taddr_s = reinterpret_cast<uint32_t *>(sm + STAGES * (A_STAGE + B_STAGE) + 128);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; s++) {
            mbar_init(full + 8 * s, 1);
            mbar_init(empty + 8 * s, 1);
        }
        for (int s = 0; s < 2; s++) {
            mbar_init(tfull + 8 * s, 1);
            mbar_init(tempty + 8 * s, 4);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         smem_u32(taddr_s))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr_s;
    const int kb_n = a.HD / BK;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < a.tiles && ok; t += gridDim.x) {
                const Tile tl = tile_of(a, t);
                const int qrow = tl.b * a.Nq + tl.m0;
                const int krow = (int)((int64_t)tl.b * a.cap + tl.n0);
                for (int kb = 0; kb < kb_n; kb++) {
                    if (!(ok = mbar_wait(empty + 8 * stage, phase ^ 1))) break;
                    mbar_expect_tx(full + 8 * stage, A_STAGE + B_STAGE);
                    tma_load_2d(a_s + stage * A_STAGE, &tmap_q, kb * BK, qrow, full + 8 * stage);
                    tma_load_2d(b_s + stage * B_STAGE, &tmap_k, kb * BK, krow, full + 8 * stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            int stage = 0, buf = 0;
            uint32_t phase = 0, tphase = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < a.tiles && ok; t += gridDim.x) {
                if (!(ok = mbar_wait(tempty + 8 * buf, tphase ^ 1))) break;
                tc_fence_after();
                const uint32_t d = tmem + buf * BN;
                for (int kb = 0; kb < kb_n; kb++) {
                    if (!(ok = mbar_wait(full + 8 * stage, phase))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < BK / 32; kk++)
                        mma_i8(d, sdesc(a_s + stage * A_STAGE + kk * 32),
                               sdesc(b_s + stage * B_STAGE + kk * 32), (kb | kk) != 0);
                    mma_commit(empty + 8 * stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                mma_commit(tfull + 8 * buf);
                if (++buf == 2) {
                    buf = 0;
                    tphase ^= 1;
                }
            }
        }
    } else {
        // ---------------- epilogue: thread = query row of the tile
        const int ew = warp & 3;  // TMEM lane quadrant this warp may access
        const int mrow = ew * 32 + lane;
        float *stg = reinterpret_cast<float *>(sm + EPI_OFF + ew * EPI_WARP);  // [32][STG_LD]
        float *scs = stg + 32 * STG_LD;                                        // [BN]
        int buf = 0;
        uint32_t tphase = 0;
        for (int64_t t = blockIdx.x; t < a.tiles; t += gridDim.x) {
            const Tile tl = tile_of(a, t);
            {
                // the tile's key scales (the same for every row), 8 per lane
                __syncwarp();  // every lane is done with the previous tile's scales
                const int64_t k0 = (int64_t)tl.n0 + 8 * lane;
                const float *src = a.kscale + (int64_t)tl.b * a.cap + k0;
                float4 s0, s1;
                if (a.vec && k0 + 8 <= a.cap) {
                    s0 = __ldg(reinterpret_cast<const float4 *>(src));
                    s1 = __ldg(reinterpret_cast<const float4 *>(src) + 1);
                } else {
                    float e[8];
#pragma unroll
                    for (int j = 0; j < 8; j++) e[j] = k0 + j < a.cap ? __ldg(src + j) : 0.0f;
                    s0 = make_float4(e[0], e[1], e[2], e[3]);
                    s1 = make_float4(e[4], e[5], e[6], e[7]);
                }
                reinterpret_cast<float4 *>(scs)[2 * lane] = s0;
                reinterpret_cast<float4 *>(scs)[2 * lane + 1] = s1;
                __syncwarp();
            }
            if (!mbar_wait(tfull + 8 * buf, tphase)) break;
            tc_fence_after();
            const int m = tl.m0 + mrow;
            const bool row_ok = m < a.Nq;
            int64_t V = 0;
            if (row_ok) {
                V = visible_len(a.ctx_len, a.q_pos, tl.b, m, a.Nq);
                if (V > a.cap) V = a.cap;
            }
            const int64_t bq = (int64_t)tl.b * a.Nq + m;
            const int64_t bq0 = (int64_t)tl.b * a.Nq + tl.m0 + ew * 32;  // row of lane 0
            const uint32_t trow = tmem + ((uint32_t)(ew * 32) << 16) + buf * BN;
            int S[32];
            tmem_ld_32x32b_x32(trow, S);
#pragma unroll 1
            for (int c = 0; c < BN / 32; c++) {
                tmem_ld_wait(S);
                const int64_t t0 = (int64_t)tl.n0 + c * 32;
                float v[32];
#pragma unroll
                for (int u = 0; u < 8; u++) {
                    const float4 sc = reinterpret_cast<const float4 *>(scs + c * 32)[u];
                    v[4 * u] = (t0 + 4 * u < V) ? __fmul_rn(__int2float_rn(S[4 * u]), sc.x) : -INFINITY;
                    v[4 * u + 1] =
                        (t0 + 4 * u + 1 < V) ? __fmul_rn(__int2float_rn(S[4 * u + 1]), sc.y) : -INFINITY;
                    v[4 * u + 2] =
                        (t0 + 4 * u + 2 < V) ? __fmul_rn(__int2float_rn(S[4 * u + 2]), sc.z) : -INFINITY;
                    v[4 * u + 3] =
                        (t0 + 4 * u + 3 < V) ? __fmul_rn(__int2float_rn(S[4 * u + 3]), sc.w) : -INFINITY;
                }
                if (c + 1 < BN / 32) {
                    tmem_ld_32x32b_x32(trow + (c + 1) * 32, S);  // overlaps the stores below
                } else {
                    // every column of this accumulator has been read: hand it back
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tempty + 8 * buf);
                }
                if (row_ok && t0 < V) {
                    // maxima of the four 8-token blocks of this row in the chunk
                    float mx[4];
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        mx[q] = v[8 * q];
#pragma unroll
                        for (int u = 1; u < 8; u++) mx[q] = fmaxf(mx[q], v[8 * q + u]);
                    }
                    float *bd = a.blk + bq * a.nblk_cap + t0 / 8;
                    if (a.vec_blk && t0 + 32 <= V) {
                        *reinterpret_cast<float4 *>(bd) = make_float4(mx[0], mx[1], mx[2], mx[3]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; q++)
                            if (t0 + 8 * q < V) bd[q] = mx[q];
                    }
                }
                if (a.tok) {
                    // transpose through shared memory: each warp store then covers
                    // 4 rows x 128 contiguous bytes
#pragma unroll
                    for (int u = 0; u < 8; u++)
                        reinterpret_cast<float4 *>(stg + lane * STG_LD)[u] =
                            make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                    __syncwarp();
                    const int64_t rem = row_ok ? V - t0 : 0;
                    const int nv_l = rem <= 0 ? 0 : (rem >= 32 ? 32 : (int)rem);
                    const int q = lane & 7;
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        const int rr = 4 * i + (lane >> 3);
                        const int nvr = __shfl_sync(0xffffffffu, nv_l, rr);
                        if (4 * q < nvr) {
                            const float4 f = reinterpret_cast<const float4 *>(stg + rr * STG_LD)[q];
                            float *dst = a.tok + (bq0 + rr) * a.cap + t0 + 4 * q;
                            if (a.vec && 4 * q + 4 <= nvr) {
                                *reinterpret_cast<float4 *>(dst) = f;
                            } else {
                                dst[0] = f.x;
                                if (4 * q + 1 < nvr) dst[1] = f.y;
                                if (4 * q + 2 < nvr) dst[2] = f.z;
                                if (4 * q + 3 < nvr) dst[3] = f.w;
                            }
                        }
                    }
                    __syncwarp();
                }
            }
            if (row_ok && tl.n0 == 0 && a.n_blk) a.n_blk[bq] = (int32_t)((V + 7) / 8);
            if (++buf == 2) {
                buf = 0;
                tphase ^= 1;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem)
                     : "memory");
    }
}

}  // namespace imma

int index_mma_wait_flag(bool clear) { return read_device_flag(imma::g_imma_error, clear); }

// Use the tensor-core scan for every multi-query call whose rows split into
// whole 128-byte stages. It reads each key tile once for all the queries of a
// sequence (the per-query scan would stream the keys once per query); with a
// few queries (speculative decode tokens) most of the 128-row query tile is
// padding, but the MMA work per key tile (about 6 us per SM) stays below the
// time to stream that tile from HBM (about 12 us), so the scan stays HBM-bound.
bool index_mma_supported(int Nq, int HD, int64_t cap, int B) {
    return Nq >= 2 && HD % imma::BK == 0 && HD <= 65536 && (int64_t)B * Nq < INT32_MAX &&
           (int64_t)B * cap < INT32_MAX;
}

int launch_index_mma(const int8_t *q, const int8_t *k, const float *kscale, const int64_t *ctx_len,
                     const int64_t *q_pos, int B, int Nq, int HD, int64_t cap, float *tok,
                     float *blk, int32_t *n_blk, cudaStream_t s) {
    using namespace imma;
    CUtensorMap mq, mk;
    if (!make_tmap_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, HD, (uint64_t)B * Nq, HD, BK, BM) ||
        !make_tmap_2d(&mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, k, HD, (uint64_t)B * cap, HD, BK, BN))
        return CSA2_ERR_CUDA;
    static PerDevice smem_set;
    if (!set_smem_limit_once(smem_set, index_mma_kernel, SMEM_BYTES)) return CSA2_ERR_CUDA;
    Args a;
    a.kscale = kscale;
    a.ctx_len = ctx_len;
    a.q_pos = q_pos;
    a.B = B;
    a.Nq = Nq;
    a.HD = HD;
    a.cap = cap;
    a.nblk_cap = (cap + 7) / 8;
    a.tok = tok;
    a.blk = blk;
    a.n_blk = n_blk;
    a.m_tiles = (Nq + BM - 1) / BM;
    a.n_tiles = (int)((cap + BN - 1) / BN);
    a.tiles = (int64_t)B * a.m_tiles * a.n_tiles;
    a.vec = (cap % 4 == 0) && aligned(kscale, 16) && (tok == nullptr || aligned(tok, 16));
    a.vec_blk = (a.nblk_cap % 4 == 0) && aligned(blk, 16);
    const int64_t grid = a.tiles < num_sms() ? a.tiles : num_sms();
    index_mma_kernel<<<(unsigned)grid, THREADS, SMEM_BYTES, s>>>(mq, mk, a);
    return launch_status();
}

}  // namespace csa2
