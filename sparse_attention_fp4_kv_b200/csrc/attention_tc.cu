// Tensor-core sparse attention for the pages' decoder shape: 64 main-Q heads,
// 512-channel shared KV head, up to 512 selected FP4 rows + 128 window rows.
//
// "890 bytes per token: how DeepSeek V4.1-Flash's KV cache works", mechanism
// 4: attention runs only over the selected candidates. "DeepSeek-V4.1-Flash:
// 890 Bytes Per Token, 437x Smaller KV Cache", CSA2 and CED sections: each
// layer has its own main Q and SWA KV; the window is the last 128 tokens.
// FP4 section of both pages: E2M1 elements with one E4M3 scale per 16 channels.
//
// One thread-block cluster of 8 CTAs (256 threads each) per query; CTA r takes
// keys [80 r, 80 r + 80) of the query's key list (selected rows, then window
// rows).
//  1. One thread issues TMA copies of the query's 64 x 512 bf16 Q and of the
//     CTA's window rows straight into 128-byte-swizzled K-major tiles (they
//     complete on an mbarrier); all threads gather the selected FP4 rows (256 B
//     of codes, 32 B of scales each) with 16-byte cp.async into a staging area.
//     The FP4 rows are then dequantized from shared memory by all 8 warps
//     (hardware E2M1 -> f16 conversion, times the E4M3 scale; exact in bf16).
//  2. One thread issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32):
//     S = Q K^T with M = 64 heads, N = 80 keys, K = 512, accumulated in TMEM.
//  3. Each of the 4 warps reads its 16 heads' logits from TMEM (two threads per
//     head), does a chunk-local softmax in fp32 and writes P to shared memory
//     as bf16 hi + lo parts (P = hi + lo to ~16 bits, so the P V product keeps
//     fp32-level accuracy with bf16 operands).
//  4. O^T = V^T P_hi^T + V^T P_lo^T: M = 128 channels (4 blocks), N = 64 heads,
//     K = 80 keys; the shared-memory KV tile is read as an MN-major A operand.
//     Accumulating O transposed keeps the MMAs at M = 128 (an M = 64 MMA runs at
//     half rate, and every tcgen05.mma has a fixed cost of about 50 cycles).
//  5. Each CTA writes its unnormalized O straight from TMEM (lane = channel, so
//     each warp store covers 128 contiguous bytes of one head), its row maxima
//     and sums into its cluster's exchange slot in the workspace (L2
//     resident); after a cluster barrier each CTA combines its 64 channels of
//     all 64 heads over the 8 partial results and writes the output. (Moving
//     the 1 MB of partials of a cluster through L2 measured about 4x faster
//     than through distributed shared memory.) Clusters are persistent over
//     query rows (at most 18, one wave on 148 SMs), so the workspace is 18
//     slots at most.
// TMEM: O^T uses columns 0..255 (all lanes); S uses lanes 16-31 of each 32-lane
// subpartition (the M = 64 accumulator layout) in columns 256..335.
// One launch per layer; scratch: one exchange slot (1.05 MB) per cluster.
#include "attention.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace csa2 {
namespace tc {

constexpr int HQ = 64;
constexpr int CH = 512;
constexpr int T = 80;        // keys per CTA
constexpr int CL = 8;        // CTAs per query (cluster size)
constexpr int THREADS = 256;
constexpr int SWA_BOX = 16;  // window rows per TMA box
constexpr int KEYS_MAX = T * CL;

constexpr int Q_CHUNK = HQ * 128;  // one 64-channel column of Q: 64 rows x 128 B
constexpr int Q_BYTES = HQ * CH * 2;
constexpr int K_CHUNK = T * 128;   // one 64-channel column of the KV tile
constexpr int K_BYTES = T * CH * 2;
constexpr int P_ATOM = HQ * 128;   // 64 tokens of P for 64 heads
constexpr int P_BYTES = 2 * P_ATOM;

constexpr int Q_OFF = 0;
constexpr int K_OFF = Q_OFF + Q_BYTES;
constexpr int PHI_OFF = K_OFF + K_BYTES;
constexpr int PLO_OFF = PHI_OFF + P_BYTES;
constexpr int M_OFF = PLO_OFF + P_BYTES;  // fp32 row max (log2 domain) [64]
constexpr int L_OFF = M_OFF + HQ * 4;     // fp32 row sum [64]
constexpr int SLOT_OFF = L_OFF + HQ * 4;  // int64 source offset per key slot [T]
constexpr int KIND_OFF = SLOT_OFF + T * 8;
constexpr int FP4_STAGE_OFF = PHI_OFF;    // raw FP4 rows [T][288], before P is written
static_assert(T * 288 <= 2 * P_BYTES, "FP4 staging must fit in the P buffers");
constexpr int BAR_OFF = (KIND_OFF + T + 15) / 16 * 16;  // [0] loads, [1] MMAs
constexpr int TADDR_OFF = BAR_OFF + 16;

constexpr int SMEM_USED = TADDR_OFF + 16;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
// Exchange slot of one cluster in the workspace: partial O [8 sources][8
// slices][64 heads][64 channels] fp32, row maxima [8][64] and row sums [8][64].
// TMEM: O^T channel block c (128 lanes x 64 heads) at columns 64 c; S (M = 64
// layout, lanes 16-31 of each quadrant) at columns S_COL..S_COL + 79.
constexpr uint32_t S_COL = 256;
constexpr int64_t XSLOT_FLOATS = (int64_t)CL * HQ * CH + 2 * CL * HQ;
// Clusters resident at once (148 SMs / 8); each walks query rows with this stride.
constexpr int MAX_CLUSTERS = 18;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

constexpr float LOG2E = 1.4426950408889634f;
constexpr long WAIT_LIMIT = 1L << 24;

__device__ int g_attn_error = 0;

// ---------------------------------------------------------------- PTX wrappers
// Bounded wait on an mbarrier phase; returns false if the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase) {
    for (long it = 0; it < WAIT_LIMIT; it++) {
        uint32_t done;
        asm volatile(
            "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            "selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(bar), "r"(phase)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_dsmem_v4(uint32_t addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}
__device__ __forceinline__ void st_dsmem_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ float4 ld_dsmem_v4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__global__ void __launch_bounds__(THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tswa,
                   AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sm = smem_raw + (base - raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_rank();

    float *m_s = reinterpret_cast<float *>(sm + M_OFF);
    float *l_s = reinterpret_cast<float *>(sm + L_OFF);
    int64_t *slot_src = reinterpret_cast<int64_t *>(sm + SLOT_OFF);
    uint8_t *slot_kind = sm + KIND_OFF;
    const uint32_t bar_ld = base + BAR_OFF, bar = base + BAR_OFF + 8;
    uint32_t *taddr_s = reinterpret_cast<uint32_t *>(sm + TADDR_OFF);
    // this cluster's exchange slot in the workspace
    float *xo = reinterpret_cast<float *>(a.ws) + (int64_t)blockIdx.y * XSLOT_FLOATS;
    float *xm = xo + CL * HQ * CH;
    float *xl = xm + CL * HQ;

    // ---- once per CTA: mbarriers and TMEM
    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tmem_alloc(base + TADDR_OFF, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr_s;
    const int64_t rows = (int64_t)a.B * a.Nq;
    uint32_t ld_phase = 0;
    bool ok = true;
    // dependency on the previous kernel of the stream: at once, or (prefetch)
    // after the first row's selected FP4 rows are gathered and dequantized
    bool waited = !a.prefetch;
    if (waited) {
        grid_dep_wait();
        grid_dep_launch();
    }

    // The cluster walks query rows blockIdx.y, blockIdx.y + gridDim.y, ...
    for (int64_t bq = blockIdx.y; bq < rows; bq += gridDim.y) {
        const int b = (int)(bq / a.Nq);
        const AttnWindow w = attn_window(a, b, bq);
        // Window slots of this CTA: [js, je) are window keys; TMA copies them in
        // boxes of SWA_BOX rows starting at js (a multiple of 16).
        const int k0 = (int)rank * T;
        int js = a.K - k0;
        js = js < 0 ? 0 : (js > T ? T : js);
        int je = a.K + w.n - k0;
        je = je < js ? js : (je > T ? T : je);
        const int nbox = (je - js + SWA_BOX - 1) / SWA_BOX;
        const int cover_end = js + nbox * SWA_BOX;  // slots written by the window boxes

        if (tid < T) {
            const int kidx = k0 + tid;
            uint8_t kind = 0;
            int64_t src = 0;
            if (kidx < a.K) {
                const int32_t pos = a.topk[bq * a.K + kidx];
                if (pos >= 0 && pos < a.cap) {
                    kind = 1;
                    src = (int64_t)b * a.cap + pos;
                }
            } else if (kidx - a.K < w.n) {
                kind = 2;
            }
            slot_kind[tid] = kind;
            slot_src[tid] = src;
        }
        if (tid == 0)
            mbar_expect_tx(bar_ld, (uint32_t)Q_BYTES + (uint32_t)nbox * 8u * SWA_BOX * 128u);
        __syncthreads();

        // ---- load phase: Q and window rows by TMA, FP4 rows by cp.async
        // slots that no copy writes (invalid keys outside the window boxes) are zeroed
        for (int i = tid; i < T * 64; i += THREADS) {
            const int j = i >> 6, pg = i & 63;
            if (slot_kind[j] == 0 && (j < js || j >= cover_end))
                st_shared_v4(base + K_OFF + (pg >> 3) * K_CHUNK + sw128(j, pg & 7),
                             make_uint4(0, 0, 0, 0));
        }
        // Q and this CTA's window rows by TMA (one thread)
        auto issue_q_swa = [&]() {
            const int qrow = (int)(bq * HQ);
#pragma unroll
            for (int cc = 0; cc < 8; cc++)
                tma_load_2d(base + Q_OFF + cc * Q_CHUNK, &tq, cc * 64, qrow, bar_ld);
            const int wrow0 = (int)((int64_t)b * a.swa_rows + w.row0 + (k0 + js - a.K));
            for (int bx = 0; bx < nbox; bx++)
#pragma unroll
                for (int cc = 0; cc < 8; cc++)
                    tma_load_2d(base + K_OFF + cc * K_CHUNK + (js + bx * SWA_BOX) * 128, &tswa,
                                cc * 64, wrow0 + bx * SWA_BOX, bar_ld);
        };
        if (waited && tid == 0) issue_q_swa();
        for (int i = tid; i < T * 18; i += THREADS) {  // (slot, 16-byte piece of its 288 B)
            const int j = i / 18, pc = i - j * 18;
            if (slot_kind[j] != 1 || (a.mx && pc == 17)) continue;  // MXFP4: 16 scale bytes
            const int64_t cell = slot_src[j];
            const uint8_t *src = pc < 16 ? a.kv_fp4 + cell * 256 + pc * 16
                                         : a.kv_sf + cell * (a.mx ? 16 : 32) + (pc - 16) * 16;
            cp_async16(base + FP4_STAGE_OFF + j * 288 + pc * 16, src);
        }
        cp_async_wait_all();
        __syncthreads();

        // ---- dequantize the FP4 rows into the KV tile (slots of kind 1; the
        // TMA copies write only window slots, so this need not wait for them)
        const uint8_t *stage = sm + FP4_STAGE_OFF;
        for (int i = tid; i < T * 32; i += THREADS) {  // (slot, 16-channel group)
            const int j = i >> 5, g = i & 31;
            if (slot_kind[j] != 1) continue;
            const uint2 codes = *reinterpret_cast<const uint2 *>(stage + j * 288 + g * 8);
            const float s = kv_group_scale(stage + j * 288 + 256, g, a.mx);
            uint32_t wds[8];
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const uint32_t byte = ((u < 4 ? codes.x : codes.y) >> (8 * (u & 3))) & 0xFF;
                const float2 f = e2m1x2_to_f32x2(byte);
                wds[u] = pack_bf16x2(f.x * s, f.y * s);
            }
            const int pg = g * 2;  // two 16-byte pieces
            const uint32_t d0 = base + K_OFF + (pg >> 3) * K_CHUNK + sw128(j, pg & 7);
            const uint32_t d1 = base + K_OFF + ((pg + 1) >> 3) * K_CHUNK + sw128(j, (pg + 1) & 7);
            st_shared_v4(d0, make_uint4(wds[0], wds[1], wds[2], wds[3]));
            st_shared_v4(d1, make_uint4(wds[4], wds[5], wds[6], wds[7]));
        }
        fence_proxy_async();
        if (!waited) {
            grid_dep_wait();
            grid_dep_launch();
            waited = true;
            if (tid == 0) issue_q_swa();
        }
        if (ok) ok = mbar_wait(bar_ld, ld_phase);
        ld_phase ^= 1;
        __syncthreads();

        // ---- S = Q K^T  (M = 64, N = 80, K = 512) into TMEM lanes 16..31
        const uint32_t s_tmem = tmem + (16u << 16) + S_COL;
        if (tid == 0 && ok) {
            tc_fence_after();
            constexpr uint32_t id_s = idesc_bf16(HQ, T, false);
#pragma unroll 1
            for (int kk = 0; kk < CH / 16; kk++) {
                const uint32_t off = (kk & 3) * 32;
                const uint64_t ad = sdesc(base + Q_OFF + (kk >> 2) * Q_CHUNK + off, 16, 1024);
                const uint64_t bd = sdesc(base + K_OFF + (kk >> 2) * K_CHUNK + off, 16, 1024);
                mma_bf16(s_tmem, ad, bd, id_s, kk > 0);
            }
            mma_commit(bar);
        }
        if (ok) ok = mbar_wait(bar, 0);
        tc_fence_after();

        // ---- softmax over this CTA's keys (warps 0-3; two threads per head)
        const int h = (warp & 3) * 16 + (lane & 15);
        const int half = lane >> 4;
        if (warp < 4) {
            const float sl2 = a.scale * LOG2E;
            float p[40];
            {
                float v32[32], v8[8];
                const uint32_t row_addr = s_tmem + ((uint32_t)(warp * 32) << 16);
                tmem_ld_16x32x2_32(row_addr + 0, v32);
                tmem_ld_16x32x2_8(row_addr + 64, v8);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int j = half * 32 + i;
                    p[i] = (ok && slot_kind[j] != 0) ? v32[i] * sl2 : -INFINITY;
                }
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const int j = 64 + half * 8 + i;
                    p[32 + i] = (ok && slot_kind[j] != 0) ? v8[i] * sl2 : -INFINITY;
                }
            }
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 40; i++) mx = fmaxf(mx, p[i]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            float sum = 0.0f;
#pragma unroll
            for (int i = 0; i < 40; i++) {
                p[i] = (p[i] == -INFINITY) ? 0.0f : ex2(p[i] - mx);
                sum += p[i];
            }
            sum += __shfl_xor_sync(0xffffffffu, sum, 16);
            if (half == 0) {
                m_s[h] = mx;
                l_s[h] = sum;
            }
            // P = hi + lo (bf16), K-major 128B-swizzled tiles: tokens 0..63 in the
            // first atom column, 64..79 in the second.
#pragma unroll
            for (int piece = 0; piece < 5; piece++) {
                const int tok0 = piece < 4 ? half * 32 + piece * 8 : 64 + half * 8;
                const float *pp = p + piece * 8;
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const __nv_bfloat162 hb = __floats2bfloat162_rn(pp[2 * u], pp[2 * u + 1]);
                    const float2 hf = __bfloat1622float2(hb);
                    hi[u] = *reinterpret_cast<const uint32_t *>(&hb);
                    lo[u] = pack_bf16x2(pp[2 * u] - hf.x, pp[2 * u + 1] - hf.y);
                }
                const uint32_t off = (tok0 >> 6) * P_ATOM + sw128(h, (tok0 & 63) >> 3);
                st_shared_v4(base + PHI_OFF + off, make_uint4(hi[0], hi[1], hi[2], hi[3]));
                st_shared_v4(base + PLO_OFF + off, make_uint4(lo[0], lo[1], lo[2], lo[3]));
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- O^T = V^T P_hi^T + V^T P_lo^T  (M = 128 channels x 4 blocks, N = 64
        // heads, K = 80 keys): V^T is the KV tile read MN-major, P^T the P tiles
        // read K-major; block c of 128 channels accumulates in columns 64 c
        if (tid == 0 && ok) {
            tc_fence_after();
            constexpr uint32_t id_o = idesc_bf16(128, HQ, false, true);
#pragma unroll 1
            for (int kk = 0; kk < T / 16; kk++) {
                const uint32_t poff = (kk >> 2) * P_ATOM + (kk & 3) * 32;
                const uint64_t phi = sdesc(base + PHI_OFF + poff, 16, 1024);
                const uint64_t plo = sdesc(base + PLO_OFF + poff, 16, 1024);
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    const uint64_t vd = sdesc(base + K_OFF + 2 * c * K_CHUNK + kk * 2048, K_CHUNK, 1024);
                    mma_bf16(tmem + 64 * c, vd, phi, id_o, kk > 0);
                    mma_bf16(tmem + 64 * c, vd, plo, id_o, 1);
                }
            }
            mma_commit(bar);
        }
        if (ok) ok = mbar_wait(bar, 1);
        tc_fence_after();

        // ---- publish this CTA's unnormalized O, row maxima and sums in the
        // cluster's exchange slot (L2), laid out [source][64-channel slice][64
        // heads][64 channels]. TMEM lane = channel, so every warp store of one
        // head writes 32 consecutive channels (128 bytes); warps w and w + 4
        // take channel blocks 0-1 and 2-3.
        {
            const int q4 = warp & 3;
            const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
#pragma unroll 1
            for (int c = 2 * (warp >> 2); c < 2 * (warp >> 2) + 2; c++) {
                const int ch = 128 * c + 32 * q4 + lane;  // this thread's channel
                float *dst = xo + ((int64_t)rank * CL + (ch >> 6)) * (HQ * 64) + (ch & 63);
#pragma unroll 1
                for (int hc = 0; hc < 2; hc++) {
                    float v[32];
                    tmem_ld_32x32b_32(lane_addr + 64 * c + 32 * hc, v);
#pragma unroll
                    for (int i = 0; i < 32; i++) dst[(32 * hc + i) * 64] = ok ? v[i] : 0.0f;
                }
            }
            if (warp < 4 && half == 0) {
                xm[rank * HQ + h] = ok ? m_s[h] : -INFINITY;
                xl[rank * HQ + h] = ok ? l_s[h] : 0.0f;
            }
        }
        __syncthreads();
        __threadfence();
        tc_fence_before();
        cluster_sync();  // all partial results of this row are in the slot

        // ---- combine: this CTA owns channels [64 rank, 64 rank + 64); the slice
        // of source r is contiguous at xo[r][rank]. Thread t takes the 16-byte
        // chunks e = 4 (t + 256 u), u = 0..3, of the [64 heads][64 channels]
        // slice.
        {
            float *wts = reinterpret_cast<float *>(sm + PHI_OFF);  // [64 heads][8] weight / den
            if (tid < HQ) {
                float mr[CL], lr[CL];
#pragma unroll
                for (int r = 0; r < CL; r++) {
                    mr[r] = __ldcg(xm + r * HQ + tid);
                    lr[r] = __ldcg(xl + r * HQ + tid);
                }
                float M = -INFINITY;
#pragma unroll
                for (int r = 0; r < CL; r++) M = fmaxf(M, mr[r]);
                float den = 0.0f, wg[CL];
#pragma unroll
                for (int r = 0; r < CL; r++) {
                    wg[r] = (M == -INFINITY || mr[r] == -INFINITY) ? 0.0f : ex2(mr[r] - M);
                    den += wg[r] * lr[r];
                }
                const float inv = den > 0.0f ? 1.0f / den : 0.0f;
#pragma unroll
                for (int r = 0; r < CL; r++) wts[tid * CL + r] = wg[r] * inv;
            }
            float4 f[4][CL];
#pragma unroll
            for (int u = 0; u < 4; u++)
#pragma unroll
                for (int r = 0; r < CL; r++)
                    f[u][r] = __ldcg(reinterpret_cast<const float4 *>(
                                         xo + ((int64_t)r * CL + rank) * (HQ * 64)) +
                                     tid + 256 * u);
            __syncthreads();  // weights ready
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int e = 4 * (tid + 256 * u);
                const int hh = e >> 6, ch = e & 63;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int r = 0; r < CL; r++) {
                    const float wr = wts[hh * CL + r];
                    acc.x += wr * f[u][r].x;
                    acc.y += wr * f[u][r].y;
                    acc.z += wr * f[u][r].z;
                    acc.w += wr * f[u][r].w;
                }
                *reinterpret_cast<float4 *>(a.out + (bq * HQ + hh) * (int64_t)CH + (int)rank * 64 + ch) =
                    acc;
            }
        }
        // the slot, the tiles and TMEM are free for the next row (after the last
        // row nothing is shared any more: the exchange went through global memory)
        if (bq + (int64_t)gridDim.y < rows) cluster_sync();
    }
    if (!ok && tid == 0) atomicExch(&g_attn_error, 1);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tc

bool attn_tc_supported(const AttnArgs &a) {
    const int nwin = a.n_win < a.swa_rows ? a.n_win : a.swa_rows;
    const bool has_win = nwin > 0 && a.swa != nullptr;
    return a.C == tc::CH && a.Hq == tc::HQ && a.K + (nwin > 0 ? nwin : 0) <= tc::KEYS_MAX &&
           a.K % 16 == 0 && aligned(a.q, 16) && aligned(a.kv_fp4, 16) && aligned(a.kv_sf, 16) &&
           (!has_win || (aligned(a.swa, 16) && (int64_t)a.B * a.swa_rows >= tc::SWA_BOX)) &&
           (int64_t)a.B * a.Nq * tc::HQ < INT32_MAX && (int64_t)a.B * a.swa_rows < INT32_MAX;
}

int launch_attn_tc(const AttnArgs &a, cudaStream_t s) {
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(tc::attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc::SMEM_BYTES) != cudaSuccess)
            return CSA2_ERR_CUDA;
        attr = true;
    }
    const int64_t rows = (int64_t)a.B * a.Nq;
    if (a.ws == nullptr) return CSA2_ERR_WORKSPACE;
    CUtensorMap tq, tswa;
    if (!make_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.q, tc::CH, (uint64_t)rows * tc::HQ,
                      tc::CH * 2, 64, 64))
        return CSA2_ERR_CUDA;
    const bool has_win = a.swa != nullptr && a.swa_rows > 0 && a.n_win > 0;
    // without a window the map is never used; describe the Q tensor instead
    if (!make_tmap_2d(&tswa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, has_win ? a.swa : a.q, tc::CH,
                      has_win ? (uint64_t)a.B * a.swa_rows : (uint64_t)rows * tc::HQ, tc::CH * 2, 64,
                      tc::SWA_BOX))
        return CSA2_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    const int64_t clusters = rows < tc::MAX_CLUSTERS ? rows : tc::MAX_CLUSTERS;
    cfg.gridDim = dim3(tc::CL, (unsigned)clusters, 1);
    cfg.blockDim = dim3(tc::THREADS, 1, 1);
    cfg.dynamicSmemBytes = tc::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr_cl[2];
    attr_cl[0].id = cudaLaunchAttributeClusterDimension;
    attr_cl[0].val.clusterDim.x = tc::CL;
    attr_cl[0].val.clusterDim.y = 1;
    attr_cl[0].val.clusterDim.z = 1;
    attr_cl[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr_cl[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr_cl;
    cfg.numAttrs = a.pdl ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, tc::attn_tc_kernel, tq, tswa, a) != cudaSuccess)
        return CSA2_ERR_CUDA;
    return launch_status();
}

}  // namespace csa2

namespace csa2 {

int attn_tc_wait_flag(bool clear) { return read_device_flag(tc::g_attn_error, clear); }

size_t attn_tc_workspace_bytes(int B, int Nq) {
    const int64_t rows = (int64_t)B * Nq;
    const int64_t clusters = rows < tc::MAX_CLUSTERS ? rows : tc::MAX_CLUSTERS;
    return (size_t)clusters * tc::XSLOT_FLOATS * sizeof(float);
}

}  // namespace csa2
