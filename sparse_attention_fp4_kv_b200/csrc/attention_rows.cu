// Tensor-core sparse attention with one CTA per query row, for calls with many
// rows (a chunked-prefill Full layer: thousands of causal queries).
//
// "890 bytes per token: how DeepSeek V4.1-Flash's KV cache works", mechanism
// 4: attention runs only over the selected candidates. "DeepSeek-V4.1-Flash:
// 890 Bytes Per Token, 437x Smaller KV Cache", CSA2 and CED sections: each
// query attends to its 512 selected main-KV rows and to its own sliding window
// of the last 128 positions. FP4 section of both pages: E2M1 elements with one
// E4M3 scale per 16 channels.
//
// With many rows there is no need to split one query over several SMs (the
// split-key cluster kernel pays an exchange of partial results per query).
// Here each persistent CTA takes whole queries and walks their keys in tiles
// of 64 with an online softmax:
//   S   = Q K^T        M = 64 heads, N = 64 keys, K = 512 channels
//   O^T += V^T P^T     M = 128 channels (x 4), N = 64 heads, K = 64 keys;
// O is accumulated transposed so that its MMAs run with M = 128; V^T is the
// bf16 KV tile read as an MN-major operand, P^T the softmax weights (bf16
// hi + lo parts, ~16 significant bits) read K-major.
// Warp roles (288 threads):
//   warps 0-3  softmax (two threads per head: tile maximum, the running
//              reference maximum, P and the row sums) and the epilogue (O^T
//              from TMEM, divided by the row sum, to global memory);
//   warps 4-7  loads: Q by TMA once per query; selected FP4 rows (codes and
//              scales) straight into registers, issued before the KV tile is
//              free, then dequantized into it (exact in bf16); the next tile's
//              indices prefetched meanwhile; window rows by TMA;
//   warp 8     one thread issues the MMAs: P V of the oldest tile whose P is
//              ready, or S of the next tile (up to two tiles ahead).
// The KV tile is double-buffered; S uses two TMEM buffers; P and O^T one.
// The reference maximum m of a head only moves when a tile's maximum exceeds
// it by more than 2^8 (then O^T is rescaled in TMEM); otherwise P may reach
// 2^8, which the fp32 accumulators absorb. Softmax is exact either way:
// out = sum_j 2^(s_j - m) V_j / sum_j 2^(s_j - m).
// Every mbarrier wait is bounded in time; a role that gives up raises the
// CTA's abort flag, after which the other roles stop waiting and the kernel
// ends with its error flag set.
#include "attention.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace csa2 {
namespace tr {

constexpr int HQ = 64;
constexpr int CH = 512;
constexpr int TK = 64;  // keys per tile
constexpr int NSOFT = 128, NLOAD = 256;
constexpr int LROWS = TK / (NLOAD / 32);  // rows of a KV tile per load warp
constexpr int THREADS = NSOFT + NLOAD + 32;
constexpr int MMA_WARP = (NSOFT + NLOAD) / 32;
constexpr int BAR_SOFT = 1, BAR_LOAD = 2;  // named barriers of the two groups

constexpr int Q_CHUNK = HQ * 128;  // one 64-channel column of Q: 64 rows x 128 B
constexpr int Q_BYTES = HQ * CH * 2;
constexpr int KT_CHUNK = TK * 128;  // one 64-channel column of a KV tile
constexpr int KT_BYTES = TK * CH * 2;
constexpr int P_BYTES = HQ * TK * 2;  // one part (hi or lo) of P: 64 heads x 64 keys

constexpr int Q_OFF = 0;
constexpr int K_OFF = Q_OFF + Q_BYTES;  // two KV tiles
constexpr int P_OFF = K_OFF + 2 * KT_BYTES;  // two P buffers, each hi then lo
constexpr int KIND_OFF = P_OFF + 4 * P_BYTES;  // uint8 [2][TK]: 0 none, 1 selected, 2 window
constexpr int ALPHA_OFF = KIND_OFF + 2 * TK; // fp32 [HQ]: rescale factor of O^T
constexpr int INVL_OFF = ALPHA_OFF + HQ * 4; // fp32 [HQ]: 1 / row sum
constexpr int BAR_OFF = INVL_OFF + HQ * 4;
enum { B_QFULL, B_QFREE, B_KFULL0, B_KFULL1, B_KFREE0, B_KFREE1, B_SFULL0, B_SFULL1, B_SFREE0,
       B_SFREE1, B_PFULL0, B_PFULL1, B_PFREE0, B_PFREE1, B_OFULL, B_OFREE, NBARS };
constexpr int TADDR_OFF = BAR_OFF + NBARS * 8;
constexpr int ABORT_OFF = TADDR_OFF + 4;
constexpr int SMEM_USED = ABORT_OFF + 4;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// TMEM columns: O^T channel block c (128 lanes x 64 heads) at 64 c; S buffer
// sb (M = 64 layout: lanes 16 sb .. 16 sb + 15 of each quadrant) at 256.
constexpr uint32_t S_COL = 256;
constexpr uint32_t TMEM_COLS = 512;

constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_LOG2 = 8.0f;
constexpr uint64_t WAIT_NS = 200ull * 1000 * 1000;

__device__ int g_attn_rows_error = 0;

// Non-blocking test and suspending try of an mbarrier phase of the given parity.
__device__ __forceinline__ bool test_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ bool try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
// try_wait with a suspend-time hint (ns): returns at the phase completion or
// after about the hint.
__device__ __forceinline__ bool try_wait_hint(uint32_t bar, uint32_t parity, uint32_t ns) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        "selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(ns)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ void raise_abort(volatile int *abort) {
    *abort = 1;
    atomicExch(&g_attn_rows_error, 1);
}
// Wait for the phase of the given parity (the thread is suspended in
// try_wait, not spinning); false at once when the CTA has aborted, or
// (raising the abort) when WAIT_NS pass.
__device__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort) {
    if (test_wait(bar, parity)) return true;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; it++) {
        if (try_wait(bar, parity)) return true;
        if (*abort) return false;
        if ((it & 15) == 0) {
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > WAIT_NS) {
                raise_abort(abort);
                return false;
            }
        }
    }
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__global__ void __launch_bounds__(THREADS, 1)
    attn_rows_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tswa,
                     AttnArgs a, int n_sel_tiles, int n_win_tiles) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sm = smem_raw + (base - raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint8_t *kinds = sm + KIND_OFF;
    float *alpha_s = reinterpret_cast<float *>(sm + ALPHA_OFF);
    float *invl_s = reinterpret_cast<float *>(sm + INVL_OFF);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + ABORT_OFF);
    const uint32_t bars = base + BAR_OFF;
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };

    if (tid == 0) {
        mbar_init(bar(B_QFULL), 1);
        mbar_init(bar(B_QFREE), 1);
        for (int i = 0; i < 2; i++) {
            mbar_init(bar(B_KFULL0 + i), 1);
            mbar_init(bar(B_KFREE0 + i), 1);
            mbar_init(bar(B_SFULL0 + i), 1);
            mbar_init(bar(B_SFREE0 + i), 4);  // one arrival per softmax warp
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(bar(B_PFULL0 + i), 1);
            mbar_init(bar(B_PFREE0 + i), 1);
        }
        mbar_init(bar(B_OFULL), 1);
        mbar_init(bar(B_OFREE), 4);  // one arrival per epilogue warp
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tmem_alloc(base + TADDR_OFF, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + TADDR_OFF);
    grid_dep_wait();
    grid_dep_launch();

    const int64_t rows = (int64_t)a.B * a.Nq;
    const int NT = n_sel_tiles + n_win_tiles;

    if (warp < NSOFT / 32) {
        // ------------------------------------------------ softmax + epilogue
        const int h = warp * 16 + (lane & 15);
        const int half = lane >> 4;
        const float sl2 = a.scale * LOG2E;
        bool ok = true;
        uint32_t g = 0, qi = 0;
        for (int64_t bq = blockIdx.x; bq < rows; bq += gridDim.x, qi++) {
            float m_ref = -INFINITY, l = 0.0f;
            for (int t = 0; t < NT; t++, g++) {
                const uint32_t gb = g & 1, gp = (g >> 1) & 1;
                ok = wait_bar(bar(B_KFULL0 + gb), gp, abort) && ok;
                ok = wait_bar(bar(B_SFULL0 + gb), gp, abort) && ok;
                tc_fence_after();
                float x[32];
                tmem_ld_16x32x2_32(tmem + ((uint32_t)(16 * gb + 32 * warp) << 16) + S_COL, x);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_SFREE0 + gb));
                const uint8_t *kd = kinds + gb * TK + half * 32;
                float mt = -INFINITY;
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    x[i] = (ok && kd[i] != 0) ? x[i] * sl2 : -INFINITY;
                    mt = fmaxf(mt, x[i]);
                }
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
                const bool need = m_ref != -INFINITY && mt > m_ref + RESCALE_LOG2;
                const float m_new = (m_ref == -INFINITY || need) ? mt : m_ref;
                const float alpha = need ? ex2(m_ref - m_new) : 1.0f;
                const bool any = named_bar_or(BAR_SOFT, NSOFT, need);
                // P buffer g & 1 is free once P V of tile g - 2 has completed
                const uint32_t pb = g & 1;
                ok = wait_bar(bar(B_PFREE0 + pb), ((g >> 1) & 1) ^ 1, abort) && ok;
                if (any && g > 0) {
                    // O^T may change only after P V of tile g - 1 has completed
                    ok = wait_bar(bar(B_PFREE0 + (pb ^ 1)), ((g - 1) >> 1) & 1, abort) && ok;
                }
                if (any) {
                    if (half == 0) alpha_s[h] = alpha;
                    named_bar_sync(BAR_SOFT, NSOFT);
                    tc_fence_after();
                    // rescale O^T: this warp's 32 channel lanes of each block
#pragma unroll 1
                    for (int c = 0; c < 4; c++)
#pragma unroll 1
                        for (int hc = 0; hc < 2; hc++) {
                            const uint32_t ta =
                                tmem + ((uint32_t)(32 * warp) << 16) + 64 * c + 32 * hc;
                            float v[32];
                            tmem_ld_32x32b_32(ta, v);
#pragma unroll
                            for (int i = 0; i < 32; i++) v[i] *= alpha_s[32 * hc + i];
                            tmem_st_32x32b_32(ta, v);
                        }
                    tmem_st_wait();
                }
                m_ref = m_new;
                l *= alpha;
                float psum = 0.0f;
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    x[i] = (x[i] == -INFINITY) ? 0.0f : ex2(x[i] - m_ref);
                    psum += x[i];
                }
                psum += __shfl_xor_sync(0xffffffffu, psum, 16);
                l += psum;
                // P (bf16 hi + lo), K-major 128-byte-swizzled rows of 64 keys
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const float p0 = x[8 * q + 2 * u], p1 = x[8 * q + 2 * u + 1];
                        const __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
                        const float2 hf = __bfloat1622float2(hb);
                        hi[u] = *reinterpret_cast<const uint32_t *>(&hb);
                        lo[u] = pack_bf16x2(p0 - hf.x, p1 - hf.y);
                    }
                    const uint32_t off = sw128(h, half * 4 + q);
                    const uint32_t pbase = base + P_OFF + pb * 2 * P_BYTES;
                    st_shared_v4(pbase + off, make_uint4(hi[0], hi[1], hi[2], hi[3]));
                    st_shared_v4(pbase + P_BYTES + off, make_uint4(lo[0], lo[1], lo[2], lo[3]));
                }
                fence_proxy_async();
                tc_fence_before();
                named_bar_sync(BAR_SOFT, NSOFT);
                if (tid == 0) mbar_arrive(bar(B_PFULL0 + pb));
            }
            // ---- epilogue of row bq: O = (O^T)^T / l
            if (half == 0) invl_s[h] = l > 0.0f ? 1.0f / l : 0.0f;
            named_bar_sync(BAR_SOFT, NSOFT);
            ok = wait_bar(bar(B_OFULL), qi & 1, abort) && ok;
            tc_fence_after();
            float *orow = a.out + bq * HQ * (int64_t)CH + 32 * warp + lane;
#pragma unroll 1
            for (int c = 0; c < 4; c++)
#pragma unroll 1
                for (int hc = 0; hc < 2; hc++) {
                    float v[32];
                    tmem_ld_32x32b_32(tmem + ((uint32_t)(32 * warp) << 16) + 64 * c + 32 * hc, v);
#pragma unroll
                    for (int i = 0; i < 32; i++) {
                        const int hh = 32 * hc + i;
                        orow[(int64_t)hh * CH + 128 * c] = ok ? v[i] * invl_s[hh] : 0.0f;
                    }
                }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_OFREE));
        }
    } else if (warp < MMA_WARP) {
        // ------------------------------------------------ loads and dequantization
        const int lt = tid - NSOFT, wl = lt >> 5;
        bool ok = true;
        uint32_t g = 0, qi = 0;
        int32_t pos_next[LROWS];
        for (int64_t bq = blockIdx.x; bq < rows; bq += gridDim.x, qi++) {
            const int b = (int)(bq / a.Nq);
            const AttnWindow w = attn_window(a, b, bq);
            if (n_sel_tiles > 0) {
#pragma unroll
                for (int u = 0; u < LROWS; u++)
                    pos_next[u] = __ldg(a.topk + bq * a.K + wl + (NLOAD / 32) * u);
            }
            if (lt == 0) {
                ok = wait_bar(bar(B_QFREE), (qi & 1) ^ 1, abort) && ok;
                if (ok) {
                    mbar_expect_tx(bar(B_QFULL), Q_BYTES);
#pragma unroll
                    for (int cc = 0; cc < 8; cc++)
                        tma_load_2d(base + Q_OFF + cc * Q_CHUNK, &tq, cc * 64, (int)(bq * HQ),
                                    bar(B_QFULL));
                }
            }
            for (int t = 0; t < NT; t++, g++) {
                const uint32_t gb = g & 1, gp = (g >> 1) & 1;
                const uint32_t kt = base + K_OFF + gb * KT_BYTES;
                if (t < n_sel_tiles) {
                    // FP4 rows of this tile into registers: warp wl takes rows wl + 8 u,
                    // lane = 16-channel group (one 256-byte code row per warp load)
                    uint2 codes[LROWS];
                    uint32_t scl[LROWS / 4] = {};
                    bool vrow[LROWS];
                    // every load is issued, all before the first use (a row that is
                    // not selected reads row 0 and is zeroed after the loads)
#pragma unroll
                    for (int u = 0; u < LROWS; u++) {
                        const int32_t pos = pos_next[u];
                        vrow[u] = pos >= 0 && pos < a.cap;
                        const int64_t src = vrow[u] ? (int64_t)b * a.cap + pos : 0;
                        codes[u] = __ldg(reinterpret_cast<const uint2 *>(a.kv_fp4 + src * 256) + lane);
                        // E4M3 of this lane's 16-channel group, or the E8M0 of its 32-channel block
                        const uint32_t sb = (uint32_t)__ldg(a.mx ? a.kv_sf + src * 16 + (lane >> 1)
                                                                 : a.kv_sf + src * 32 + lane);
                        scl[u >> 2] |= sb << (8 * (u & 3));
                    }
#pragma unroll
                    for (int u = 0; u < LROWS; u++) {
                        if (!vrow[u]) {
                            codes[u] = make_uint2(0, 0);
                            scl[u >> 2] &= ~(0xFFu << (8 * (u & 3)));
                        }
                    }
                    // indices of the next selected tile, while these loads are in flight
                    if (t + 1 < n_sel_tiles) {
#pragma unroll
                        for (int u = 0; u < LROWS; u++)
                            pos_next[u] =
                                __ldg(a.topk + bq * a.K + (t + 1) * TK + wl + (NLOAD / 32) * u);
                    }
                    ok = wait_bar(bar(B_KFREE0 + gb), gp ^ 1, abort) && ok;
                    if (lane == 0) {
#pragma unroll
                        for (int u = 0; u < LROWS; u++)
                            kinds[gb * TK + wl + (NLOAD / 32) * u] = vrow[u] ? 1 : 0;
                    }
                    // even and odd channel blocks store their two 16-byte halves in
                    // opposite order, so each warp store covers all 8 bank groups
                    const int pg = 2 * lane;
                    const bool swap = ((pg >> 3) & 1) != 0;
#pragma unroll
                    for (int u = 0; u < LROWS; u++) {
                        const int j = wl + (NLOAD / 32) * u;
                        const uint32_t sc = (scl[u >> 2] >> (8 * (u & 3))) & 0xFF;
                        const float s = a.mx ? e8m0_to_f32(sc) : e4m3_to_f32(sc);
                        uint32_t wds[8];
#pragma unroll
                        for (int e = 0; e < 8; e++) {
                            const uint32_t byte =
                                ((e < 4 ? codes[u].x : codes[u].y) >> (8 * (e & 3))) & 0xFF;
                            const float2 f = e2m1x2_to_f32x2(byte);
                            wds[e] = pack_bf16x2(f.x * s, f.y * s);
                        }
                        const uint4 w0 = make_uint4(wds[0], wds[1], wds[2], wds[3]);
                        const uint4 w1 = make_uint4(wds[4], wds[5], wds[6], wds[7]);
                        const uint32_t d0 = kt + (pg >> 3) * KT_CHUNK + sw128(j, pg & 7);
                        const uint32_t d1 = kt + ((pg + 1) >> 3) * KT_CHUNK + sw128(j, (pg + 1) & 7);
                        st_shared_v4(swap ? d1 : d0, swap ? w1 : w0);
                        st_shared_v4(swap ? d0 : d1, swap ? w0 : w1);
                    }
                    fence_proxy_async();
                    named_bar_sync(BAR_LOAD, NLOAD);
                    if (lt == 0) mbar_arrive(bar(B_KFULL0 + gb));
                } else {
                    ok = wait_bar(bar(B_KFREE0 + gb), gp ^ 1, abort) && ok;
                    const int w0 = (t - n_sel_tiles) * TK;  // first window slot of this tile
                    if (lt < TK) kinds[gb * TK + lt] = (w0 + lt < w.n) ? 2 : 0;
                    named_bar_sync(BAR_LOAD, NLOAD);
                    if (lt == 0) {
                        if (ok) {
                            mbar_expect_tx(bar(B_KFULL0 + gb), KT_BYTES);
                            const int r0 = (int)((int64_t)b * a.swa_rows + w.row0 + w0);
#pragma unroll
                            for (int cc = 0; cc < 8; cc++)
                                tma_load_2d(kt + cc * KT_CHUNK, &tswa, cc * 64, r0,
                                            bar(B_KFULL0 + gb));
                        } else {
                            mbar_arrive(bar(B_KFULL0 + gb));
                        }
                    }
                }
            }
        }
    } else if (lane == 0) {
        // ------------------------------------------------ MMA issue: P V of the
        // oldest tile whose P is ready, or S of the next tile once its KV tile and
        // S buffer are (S may run up to two tiles ahead of P V)
        constexpr uint32_t id_s = idesc_bf16(HQ, TK, false);
        constexpr uint32_t id_o = idesc_bf16(128, HQ, false, true);
        // descriptors of the tile bases; an address offset adds (offset >> 4)
        const uint64_t dq = sdesc(base + Q_OFF, 16, 1024);
        const uint64_t dk0 = sdesc(base + K_OFF, 16, 1024);
        const uint64_t dv0 = sdesc(base + K_OFF, KT_CHUNK, 1024);
        const uint64_t dp0 = sdesc(base + P_OFF, 16, 1024);
        const int64_t nrows = rows > blockIdx.x ? (rows - 1 - blockIdx.x) / gridDim.x + 1 : 0;
        const int64_t total = nrows * NT;
        int64_t s_next = 0, p_next = 0;
        uint64_t last = globaltimer_ns();
        while (p_next < total && !*abort) {
            bool progressed = false;
            const bool s_cand = s_next < total && s_next < p_next + 2;
            if (p_next < s_next) {
                const int tp = (int)(p_next % NT);
                const uint32_t qp = (uint32_t)(p_next / NT);
                const uint32_t pb = (uint32_t)(p_next & 1), pp = (uint32_t)((p_next >> 1) & 1);
                // suspend here briefly only when no S is waiting to be issued
                const bool pready = s_cand ? test_wait(bar(B_PFULL0 + pb), pp)
                                           : try_wait_hint(bar(B_PFULL0 + pb), pp, 1000);
                if (pready && (tp != 0 || test_wait(bar(B_OFREE), (qp & 1) ^ 1))) {
                    tc_fence_after();
                    const uint64_t dv = dv0 + (uint64_t)((pb * KT_BYTES) >> 4);
                    const uint64_t dphi = dp0 + (uint64_t)((pb * 2 * P_BYTES) >> 4);
                    const uint64_t dplo = dphi + (uint64_t)(P_BYTES >> 4);
#pragma unroll
                    for (int kk = 0; kk < TK / 16; kk++)
#pragma unroll
                        for (int c = 0; c < 4; c++) {
                            const uint64_t vd = dv + (uint64_t)((2 * c * KT_CHUNK + kk * 2048) >> 4);
                            mma_bf16(tmem + 64 * c, vd, dphi + (uint64_t)(kk * 2), id_o,
                                     (tp > 0 || kk > 0) ? 1u : 0u);
                            mma_bf16(tmem + 64 * c, vd, dplo + (uint64_t)(kk * 2), id_o, 1u);
                        }
                    mma_commit(bar(B_KFREE0 + pb));
                    mma_commit(bar(B_PFREE0 + pb));
                    if (tp == NT - 1) mma_commit(bar(B_OFULL));
                    p_next++;
                    progressed = true;
                }
            }
            if (!progressed && s_cand) {
                const int ts = (int)(s_next % NT);
                const uint32_t qs = (uint32_t)(s_next / NT);
                const uint32_t gb = (uint32_t)(s_next & 1), gp = (uint32_t)((s_next >> 1) & 1);
                // the KV tile is usually the last to be ready: suspend on it
                if ((ts != 0 || test_wait(bar(B_QFULL), qs & 1)) &&
                    test_wait(bar(B_SFREE0 + gb), gp ^ 1) &&
                    try_wait_hint(bar(B_KFULL0 + gb), gp, p_next < s_next ? 200 : 1000)) {
                    tc_fence_after();
                    const uint64_t dk = dk0 + (uint64_t)((gb * KT_BYTES) >> 4);
                    const uint32_t sd = tmem + ((16u * gb) << 16) + S_COL;
#pragma unroll
                    for (int kk = 0; kk < CH / 16; kk++) {
                        const uint32_t off = (uint32_t)((kk >> 2) * Q_CHUNK + (kk & 3) * 32) >> 4;
                        mma_bf16(sd, dq + off, dk + off, id_s, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(B_SFULL0 + gb));
                    if (ts == NT - 1) mma_commit(bar(B_QFREE));
                    s_next++;
                    progressed = true;
                }
            }
            if (progressed) {
                last = globaltimer_ns();
            } else if (globaltimer_ns() - last > WAIT_NS) {
                raise_abort(abort);
            }
        }
    }
    __syncthreads();
    if (*abort) {
        if (tid == 0 && a.err) atomicExch(a.err, 1);
        // let copies and MMAs still in flight land before the CTA's memory is released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace tr

int attn_rows_wait_flag(bool clear) { return read_device_flag(tr::g_attn_rows_error, clear); }

bool attn_rows_supported(const AttnArgs &a) {
    const int nwin = a.n_win < a.swa_rows ? a.n_win : a.swa_rows;
    const bool has_win = nwin > 0 && a.swa != nullptr;
    return a.C == tr::CH && a.Hq == tr::HQ && a.K % tr::TK == 0 && a.K + (has_win ? nwin : 0) > 0 &&
           aligned(a.q, 16) && aligned(a.kv_fp4, 16) && aligned(a.kv_sf, 16) &&
           (!has_win || (aligned(a.swa, 16) && (int64_t)a.B * a.swa_rows >= tr::TK)) &&
           (int64_t)a.B * a.Nq * tr::HQ < INT32_MAX && (int64_t)a.B * a.swa_rows < INT32_MAX;
}

int launch_attn_rows(const AttnArgs &a, cudaStream_t s) {
    static PerDevice smem_set;
    if (!set_smem_limit_once(smem_set, tr::attn_rows_kernel, tr::SMEM_BYTES)) return CSA2_ERR_CUDA;
    const int64_t rows = (int64_t)a.B * a.Nq;
    const int nwin = a.n_win < a.swa_rows ? a.n_win : a.swa_rows;
    const bool has_win = nwin > 0 && a.swa != nullptr;
    const int n_sel_tiles = a.K / tr::TK;
    const int n_win_tiles = has_win ? (nwin + tr::TK - 1) / tr::TK : 0;
    CUtensorMap tq, tswa;
    if (!make_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.q, tr::CH, (uint64_t)rows * tr::HQ,
                      tr::CH * 2, 64, 64))
        return CSA2_ERR_CUDA;
    // without a window the map is never used; describe the Q tensor instead
    if (!make_tmap_2d(&tswa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, has_win ? a.swa : a.q, tr::CH,
                      has_win ? (uint64_t)a.B * a.swa_rows : (uint64_t)rows * tr::HQ, tr::CH * 2, 64,
                      tr::TK))
        return CSA2_ERR_CUDA;
    const int64_t grid = rows < num_sms() ? rows : num_sms();
    return launch_kernel(a.pdl, tr::attn_rows_kernel, dim3((unsigned)grid), dim3(tr::THREADS),
                         tr::SMEM_BYTES, s, tq, tswa, a, n_sel_tiles, n_win_tiles);
}

}  // namespace csa2
