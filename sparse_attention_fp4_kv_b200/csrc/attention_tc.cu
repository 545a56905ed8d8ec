// Tensor-core sparse attention for the pages' decoder shape: 64 main-Q heads,
// 512-channel shared KV head, up to 512 selected FP4 rows + 128 window rows.
//
// "890 bytes per token: how DeepSeek V4.1-Flash's KV cache works", mechanism
// 4: attention runs only over the selected candidates. "DeepSeek-V4.1-Flash:
// 890 Bytes Per Token, 437x Smaller KV Cache", CSA2 and CED sections: each
// layer has its own main Q and SWA KV; the window is the last 128 tokens.
// FP4 section of both pages: E2M1 elements with one E4M3 scale per 16 channels.
//
// One thread-block cluster of 8 CTAs (256 threads each) per (query row, head
// group); CTA r takes keys [80 r, 80 r + 80) of the row's key list (selected
// rows, then window rows) for the group's HPC heads. With few rows the 64
// heads are split into groups of 16 or 32 (HPC), so that more SMs share the
// row and each CTA's partial result is smaller; with many rows a cluster takes
// all 64 heads and loops over rows.
//  1. All threads gather the CTA's selected FP4 rows (256 B of codes, 32 B of
//     scales each) straight into registers, 16-byte loads all issued before
//     the first use, and dequantize them into the 128-byte-swizzled K-major KV
//     tile (hardware E2M1 -> f16 conversion, times the E4M3 scale; exact in
//     bf16). One thread issues TMA copies of the group's HPC x 512 bf16 Q rows
//     and of the CTA's window rows, which complete on an mbarrier.
//  2. One thread issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32):
//     S = Q K^T with M = 64 (HPC real heads), N = 80 keys, K = 512 in TMEM.
//  3. HPC / 16 warps read the heads' logits from TMEM (two threads per head),
//     do a chunk-local softmax in fp32 and write P to shared memory as bf16 hi
//     + lo parts (P = hi + lo to ~16 bits, so the P V product keeps fp32-level
//     accuracy with bf16 operands).
//  4. O^T = V^T [P_hi; P_lo]^T: M = 128 channels (4 blocks), N = 2 HPC (the
//     hi rows then the lo rows of P, one MMA for both parts), K = 80 keys; the
//     shared-memory KV tile is read as an MN-major A operand. Accumulating O
//     transposed keeps the MMAs at M = 128 (an M = 64 MMA runs at half rate,
//     and every tcgen05.mma has a fixed cost of about 50 cycles); stacking the
//     two parts of P halves their count. The epilogue adds the two halves.
//  5. Each CTA writes its unnormalized O straight from TMEM (lane = channel, so
//     each warp store covers 128 contiguous bytes of one head), its row maxima
//     and sums into its cluster's exchange slot in the workspace (L2
//     resident); after a cluster barrier each CTA combines its 64 channels of
//     the group's heads over the 8 partial results and writes the output.
//     (Moving the partials through L2 measured about 4x faster than through
//     distributed shared memory.) Clusters are persistent over (row, group)
//     items, at most as many as can be resident at once (and at most 18), so
//     the workspace is 18 slots at most.
// TMEM: O^T block c at columns 2 HPC c (hi part) and 2 HPC c + HPC (lo part),
// all lanes; S uses lanes 16-31 of each 32-lane subpartition (the M = 64
// accumulator layout) from column S_COL, which may overlap O^T columns: S is
// read by the softmax before the P V MMAs that write them are issued.
//
// Layer groups. A launch runs the attention of one group of layers that share
// the same selected rows: a Full or Reindex layer and the Reuse layers that
// follow it ("DeepSeek-V4.1-Flash", CSA2 section). Each layer has its own Q and
// window rows. A cluster that holds one (row, head group) item keeps its
// dequantized selected rows in shared memory for every layer of the group; per
// layer it copies only the layer's Q and window rows. Layer l + 1 of a query
// row starts once every CTA of that row has written layer l's output (a
// per-row counter in global memory, release/acquire, every wait bounded): the
// rows of a batch are independent sequences, so one row never waits for
// another.
#include <cstring>

#include "attention.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace csa2 {
namespace tc {

constexpr int HQ = 64;
constexpr int CH = 512;
constexpr int T = 80;        // keys per CTA
constexpr int CL = 8;        // CTAs per (row, head group) (cluster size)
constexpr int THREADS = 256;
constexpr int SWA_BOX = 8;   // window rows per TMA box
constexpr int KEYS_MAX = T * CL;
constexpr int K_CHUNK = T * 128;   // one 64-channel column of the KV tile
constexpr int K_BYTES = T * CH * 2;
constexpr int GATHER_PER_THREAD = T * 16 / THREADS;  // (slot, 32-channel group) items
static_assert(GATHER_PER_THREAD * THREADS == T * 16, "gather split");
constexpr int MAX_CLUSTERS = 18;
constexpr int MAXL = kMaxGroupLayers;  // layers per launch
constexpr float LOG2E = 1.4426950408889634f;
constexpr uint64_t WAIT_NS = 200ull * 1000 * 1000;

// Shared-memory layout and TMEM columns of a CTA that takes HPC heads.
template <int HPC>
struct Cfg {
    static constexpr int HG = HQ / HPC;            // head groups per row
    static constexpr int Q_CHUNK = HPC * 128;      // one 64-channel column of Q
    static constexpr int Q_BYTES = HPC * CH * 2;
    // P tile: per 64-token atom column, the hi rows of the HPC heads then
    // their lo rows (2 HPC rows of 128 bytes); two atom columns (80 tokens)
    static constexpr int P_ATOM = 2 * HPC * 128;
    static constexpr int P_BYTES = 2 * P_ATOM;
    static constexpr int Q_OFF = 0;
    // S is an M = 64 MMA: its A operand spans 64 rows of each Q column, of
    // which rows HPC..63 run on into the next columns and (for the last column)
    // the KV tile. Those rows only produce accumulator rows that are never
    // read, and they stay inside this CTA's shared memory.
    static constexpr int K_OFF = Q_OFF + Q_BYTES;
    static constexpr int P_OFF = K_OFF + K_BYTES;
    static constexpr int M_OFF = P_OFF + P_BYTES;    // fp32 row max (log2 domain) [HPC]
    static constexpr int L_OFF = M_OFF + HPC * 4;    // fp32 row sum [HPC]
    static constexpr int SLOT_OFF = L_OFF + HPC * 4; // int64 source row per key slot [T]
    static constexpr int KIND_OFF = SLOT_OFF + T * 8;
    // mbarriers: [0] loads, [1] MMAs, [2] the P V MMAs of channel blocks 0-1
    static constexpr int BAR_OFF = (KIND_OFF + T + 15) / 16 * 16;
    static constexpr int TADDR_OFF = BAR_OFF + 24;
    static constexpr int SMEM_USED = TADDR_OFF + 16;
    static constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
    static constexpr int MIN_BLOCKS = SMEM_BYTES <= 112 * 1024 ? 2 : 1;
    static constexpr uint32_t S_COL = HPC == 64 ? 256 : 128;
    static constexpr uint32_t TMEM_COLS = HPC == 64 ? 512 : 256;
    static constexpr uint32_t O_COLS = 8 * HPC;      // 4 channel blocks x (hi, lo) x HPC
    static constexpr int64_t XSLOT_FLOATS = (int64_t)CL * HPC * CH + 2 * CL * HPC;
    static_assert(64 * 128 <= Q_BYTES - 7 * Q_CHUNK + K_BYTES, "S A-operand rows inside the CTA");
    static_assert(O_COLS <= TMEM_COLS && S_COL + T <= TMEM_COLS, "TMEM columns");
    static_assert(HPC * CL * 4 <= P_BYTES, "combine weights fit in the P tiles");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

__device__ int g_attn_error = 0;

// The layers of one launch: per layer its Q and window tensors (as TMA maps and
// pointers) and its output. row_done (with n > 1) holds one counter per query
// row, row_base at launch: every CTA of the row adds 1 after writing its part
// of each layer's output, so layer l of the row is complete once the counter
// reaches row_base + (l + 1) x (CTAs per row).
struct alignas(64) TcLayers {
    CUtensorMap tq[MAXL];
    CUtensorMap tswa[MAXL];
    const void *q[MAXL];
    const void *swa[MAXL];
    float *out[MAXL];
    int *row_done;
    int row_base;
    int n;
};

__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_gpu_add(int *p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Waits (one thread) until *p >= target; false after limit_ns of global time.
__device__ __forceinline__ bool wait_counter_bounded(const int *p, int target, uint64_t limit_ns) {
    uint64_t t0 = 0;
    for (;;) {
        if (ld_acquire_gpu(p) >= target) return true;
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) {
            t0 = now;
        } else if (now - t0 > limit_ns) {
            return false;
        }
        __nanosleep(64);
    }
}

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// O^T columns [col, col + HPC) of the 32 lanes of this warp's subpartition
// into v[0..HPC) (HPC = 16, 32 or 64).
template <int HPC>
__device__ __forceinline__ void load_ot(uint32_t taddr, float (&v)[HPC]) {
    if constexpr (HPC == 16) {
        tmem_ld_32x32b_16(taddr, v);
    } else {
#pragma unroll
        for (int hc = 0; hc < HPC / 32; hc++) {
            float w[32];
            tmem_ld_32x32b_32(taddr + 32 * hc, w);
#pragma unroll
            for (int i = 0; i < 32; i++) v[32 * hc + i] = w[i];
        }
    }
}

// Slots of a CTA: [0, ks) for its ks selected keys, [ks, ks + wsz) for its wsz
// window rows (ks and wsz multiples of 8, ks + wsz <= T).
template <int HPC>
__global__ void __launch_bounds__(THREADS, Cfg<HPC>::MIN_BLOCKS)
    attn_tc_kernel(const __grid_constant__ TcLayers lay, AttnArgs a, int ks, int wsz) {
    using L = Cfg<HPC>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sm = smem_raw + (base - raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_rank();

    float *m_s = reinterpret_cast<float *>(sm + L::M_OFF);
    float *l_s = reinterpret_cast<float *>(sm + L::L_OFF);
    int64_t *slot_src = reinterpret_cast<int64_t *>(sm + L::SLOT_OFF);
    uint8_t *slot_kind = sm + L::KIND_OFF;
    const uint32_t bar_ld = base + L::BAR_OFF, bar = base + L::BAR_OFF + 8;
    const uint32_t bar_pv = base + L::BAR_OFF + 16;
    uint32_t *taddr_s = reinterpret_cast<uint32_t *>(sm + L::TADDR_OFF);
    // this cluster's exchange slot in the workspace
    float *xo = reinterpret_cast<float *>(a.ws) + (int64_t)blockIdx.y * L::XSLOT_FLOATS;
    float *xm = xo + CL * HPC * CH;
    float *xl = xm + CL * HPC;

    // ---- once per CTA: mbarriers and TMEM
    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar, 1);
        mbar_init(bar_pv, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tmem_alloc(base + L::TADDR_OFF, L::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *taddr_s;
    const int64_t rows = (int64_t)a.B * a.Nq;
    const int64_t items = rows * L::HG;
    const int NL = lay.n;
    // A cluster with at most one item keeps its dequantized selected rows for
    // every layer. With 64 heads per cluster a cluster owns whole rows, so it
    // takes its rows one after another and runs all layers of a row before the
    // next (row_major): one gather per row, and layer l + 1 of the row follows
    // layer l through the cluster barrier, not the per-row counters. Otherwise
    // (several head groups per row, more items than clusters) the cluster
    // walks its items layer by layer and gathers per item and layer.
    const bool keep = (int64_t)gridDim.y >= items;
    const bool row_major = L::HG == 1;
    const int64_t n_mine =
        (int64_t)blockIdx.y < items ? (items - 1 - (int64_t)blockIdx.y) / gridDim.y + 1 : 0;
    uint32_t ld_phase = 0, pv_phase = 0;
    bool ld_pending = false;  // (thread 0) copies issued on bar_ld and not yet waited for
    bool ok = true;
    // Q and window rows of this cluster's first item, every layer: warmed in
    // L2 before the dependency wait (a prefetch only moves data into L2; the
    // copies that read it come after the wait, and for layer l + 1 after the
    // row's layer-l output). In a decoder these inputs are written just before
    // the layer runs and are L2-resident then.
    if (tid == 32 && (int64_t)blockIdx.y < items) {
        const int64_t bq0 = (int64_t)blockIdx.y / L::HG;
        const int hg0 = (int)((int64_t)blockIdx.y - bq0 * L::HG);
        const int b0 = (int)(bq0 / a.Nq);
        const AttnWindow w = attn_window(a, b0, bq0);
        const int w0 = (int)rank * wsz;
        int wn = w.n - w0;
        wn = wn < 0 ? 0 : (wn > wsz ? wsz : wn);
        for (int l = 0; l < NL; l++) {
            bulk_prefetch_l2(static_cast<const uint8_t *>(lay.q[l]) +
                                 (bq0 * HQ + hg0 * HPC) * (int64_t)CH * 2,
                             (uint32_t)(HPC * CH * 2));
            if (wn > 0)
                bulk_prefetch_l2(static_cast<const uint8_t *>(lay.swa[l]) +
                                     ((int64_t)b0 * a.swa_rows + w.row0 + w0) * CH * 2,
                                 (uint32_t)(wn * CH * 2));
        }
    }
    // dependency on the previous kernel of the stream: at once, or (prefetch)
    // after the first item's selected FP4 rows are gathered and dequantized
    bool waited = !a.prefetch;
    if (waited) {
        grid_dep_wait();
        grid_dep_launch();
    }

    // The cluster's (row, head group) items are blockIdx.y, blockIdx.y +
    // gridDim.y, ... (with keep, just one). Step s is (layer, item) in layer
    // order, or with row_major (item, layer) in item order.
    for (int64_t step = 0; step < n_mine * NL; step++) {
        const int l = row_major ? (int)(step % NL) : (int)(step / n_mine);
        const int64_t it = (int64_t)blockIdx.y + (row_major ? step / NL : step % n_mine) * gridDim.y;
        const bool gather = (l == 0) || (!keep && !row_major);
        {
            const int64_t bq = it / L::HG;
            const int hg = (int)(it - bq * L::HG);
            const int b = (int)(bq / a.Nq);
            const AttnWindow w = attn_window(a, b, bq);
            // CTA r takes selected keys [r ks, r ks + ks) and window rows
            // [r wsz, r wsz + wsz), so that every CTA gathers about as many FP4
            // rows and copies about as many window rows. The window rows arrive
            // by TMA in boxes of SWA_BOX rows from slot ks; slots [ks, cover_end)
            // are written by the boxes.
            const int w0 = (int)rank * wsz;
            int wn = w.n - w0;
            wn = wn < 0 ? 0 : (wn > wsz ? wsz : wn);
            const int js = ks;
            const int nbox = (wn + SWA_BOX - 1) / SWA_BOX;
            const int cover_end = js + nbox * SWA_BOX;

            if (gather && tid < T) {
                uint8_t kind = 0;
                int64_t src = 0;
                if (tid < ks) {
                    const int kidx = (int)rank * ks + tid;
                    if (kidx < a.K) {
                        const int32_t pos = a.topk[bq * a.K + kidx];
                        if (pos >= 0 && pos < a.cap) {
                            kind = 1;
                            src = (int64_t)b * a.cap + pos;
                        }
                    }
                } else if (tid - ks < wn) {
                    kind = 2;
                }
                slot_kind[tid] = kind;
                slot_src[tid] = src;
            }
            // layer l of this row follows layer l - 1 of the same row: every
            // CTA of the row has written its part of that output (with
            // row_major this cluster wrote all of it, before its last barrier)
            if (l > 0 && !row_major && tid == 0 && ok)
                ok = wait_counter_bounded(lay.row_done + bq, lay.row_base + l * L::HG * CL, WAIT_NS);
            if (tid == 0)
                mbar_expect_tx(bar_ld, (uint32_t)L::Q_BYTES + (uint32_t)nbox * 8u * SWA_BOX * 128u);
            __syncthreads();

            // Q rows of the group and this CTA's window rows by TMA (one thread)
            auto issue_q_swa = [&]() {
                const int qrow = (int)(bq * HQ + hg * HPC);
#pragma unroll
                for (int cc = 0; cc < 8; cc++)
                    tma_load_2d(base + L::Q_OFF + cc * L::Q_CHUNK, &lay.tq[l], cc * 64, qrow, bar_ld);
                const int wrow0 = (int)((int64_t)b * a.swa_rows + w.row0 + w0);
                for (int bx = 0; bx < nbox; bx++)
#pragma unroll
                    for (int cc = 0; cc < 8; cc++)
                        tma_load_2d(base + L::K_OFF + cc * K_CHUNK + (js + bx * SWA_BOX) * 128,
                                    &lay.tswa[l], cc * 64, wrow0 + bx * SWA_BOX, bar_ld);
            };
            if (waited && tid == 0 && ok) {
                issue_q_swa();
                ld_pending = true;
            }

            // ---- selected FP4 rows: codes and scales into registers (all loads
            // first, unconditionally: a slot without a selected row reads row 0),
            // then dequantized into the KV tile. Item i = (slot i / 16, 32-channel
            // group i % 16): 16 bytes of codes and the group's two E4M3 scales
            // (one E8M0 with MXFP4); a warp reads two rows' 256 code bytes. Slots
            // that no copy writes (invalid keys outside the window boxes) are
            // zeroed; the TMA copies write only window slots, so this need not
            // wait for them.
            if (gather) {
                uint4 codes[GATHER_PER_THREAD];
                uint32_t sfb[GATHER_PER_THREAD];
#pragma unroll
                for (int u = 0; u < GATHER_PER_THREAD; u++) {
                    const int i = tid + THREADS * u, j = i >> 4, gp = i & 15;
                    const int64_t cell = slot_src[j];
                    codes[u] = __ldcg(reinterpret_cast<const uint4 *>(a.kv_fp4 + cell * 256) + gp);
                    sfb[u] = a.mx ? (uint32_t)__ldcg(a.kv_sf + cell * 16 + gp)
                                  : (uint32_t)__ldcg(
                                        reinterpret_cast<const unsigned short *>(a.kv_sf + cell * 32) + gp);
                }
#pragma unroll
                for (int u = 0; u < GATHER_PER_THREAD; u++) {
                    const int i = tid + THREADS * u, j = i >> 4, gp = i & 15;
                    const int kind = slot_kind[j];
                    if (kind == 2 || (kind == 0 && j >= js && j < cover_end)) continue;
                    uint32_t wds[16];
                    if (kind == 1) {
                        // channels 32 gp .. 32 gp + 15 take the first scale, the rest the second
                        const float s0 = a.mx ? e8m0_to_f32(sfb[u]) : e4m3_to_f32(sfb[u] & 0xFF);
                        const float s1 = a.mx ? s0 : e4m3_to_f32(sfb[u] >> 8);
                        const uint32_t cw[4] = {codes[u].x, codes[u].y, codes[u].z, codes[u].w};
#pragma unroll
                        for (int e = 0; e < 16; e++) {
                            const uint32_t byte = (cw[e >> 2] >> (8 * (e & 3))) & 0xFF;
                            const float2 f = e2m1x2_to_f32x2(byte);
                            const float sc = e < 8 ? s0 : s1;
                            wds[e] = pack_bf16x2(f.x * sc, f.y * sc);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; e++) wds[e] = 0u;
                    }
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        const int pg = gp * 4 + q;  // 16-byte piece (8 channels) of the row
                        st_shared_v4(base + L::K_OFF + (pg >> 3) * K_CHUNK + sw128(j, pg & 7),
                                     make_uint4(wds[4 * q], wds[4 * q + 1], wds[4 * q + 2], wds[4 * q + 3]));
                    }
                }
                fence_proxy_async();
            }
            if (!waited) {
                grid_dep_wait();
                grid_dep_launch();
                waited = true;
                if (tid == 0 && ok) {
                    issue_q_swa();
                    ld_pending = true;
                }
            }
            if (tid == 0 && ld_pending) {
                ok = mbar_wait_bounded(bar_ld, ld_phase, WAIT_NS);
                ld_pending = !ok;   // a copy that did not complete is drained at exit
            }
            if (!ld_pending) ld_phase ^= 1;
            ok = __syncthreads_and(ok) != 0;

            // ---- S = Q K^T  (M = 64, N = 80, K = 512) into TMEM lanes 16..31
            const uint32_t s_tmem = tmem + (16u << 16) + L::S_COL;
            if (tid == 0 && ok) {
                tc_fence_after();
                constexpr uint32_t id_s = idesc_bf16(64, T, false);
#pragma unroll 1
                for (int kk = 0; kk < CH / 16; kk++) {
                    const uint32_t off = (kk & 3) * 32;
                    const uint64_t ad = sdesc(base + L::Q_OFF + (kk >> 2) * L::Q_CHUNK + off, 16, 1024);
                    const uint64_t bd = sdesc(base + L::K_OFF + (kk >> 2) * K_CHUNK + off, 16, 1024);
                    mma_bf16(s_tmem, ad, bd, id_s, kk > 0);
                }
                mma_commit(bar);
            }

            // ---- softmax over this CTA's keys (warps 0 .. HPC/16 - 1; two threads per head)
            const int h = warp * 16 + (lane & 15);
            const int half = lane >> 4;
            if (warp < HPC / 16) {
                if (ok) ok = mbar_wait_bounded(bar, 0, WAIT_NS);
                tc_fence_after();
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
                // P = hi + lo (bf16), K-major 128B-swizzled tiles: tokens 0..63 in
                // the first atom column, 64..79 in the second; head h's hi part in
                // row h, its lo part in row HPC + h.
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
                    const uint32_t atom = base + L::P_OFF + (tok0 >> 6) * L::P_ATOM;
                    st_shared_v4(atom + sw128(h, (tok0 & 63) >> 3), make_uint4(hi[0], hi[1], hi[2], hi[3]));
                    st_shared_v4(atom + sw128(HPC + h, (tok0 & 63) >> 3),
                                 make_uint4(lo[0], lo[1], lo[2], lo[3]));
                }
                fence_proxy_async();
                tc_fence_before();
            }
            ok = __syncthreads_and(ok) != 0;

            // ---- O^T = V^T [P_hi; P_lo]^T  (M = 128 channels x 4 blocks, N = 2 HPC,
            // K = 80 keys): V^T is the KV tile read MN-major, [P_hi; P_lo]^T the P
            // tile read K-major; block c of 128 channels accumulates in columns
            // [2 HPC c, 2 HPC c + 2 HPC) (hi part, then lo part)
            // Channel blocks 0-1 first, committed on their own barrier, so that
            // warps 0-3 publish them while blocks 2-3 are multiplied.
            const bool pv_issued = ok;  // uniform here
            if (tid == 0 && ok) {
                tc_fence_after();
                constexpr uint32_t id_o = idesc_bf16(128, 2 * HPC, false, true);
#pragma unroll
                for (int c2 = 0; c2 < 2; c2++) {
#pragma unroll 1
                    for (int kk = 0; kk < T / 16; kk++) {
                        const uint64_t pd =
                            sdesc(base + L::P_OFF + (kk >> 2) * L::P_ATOM + (kk & 3) * 32, 16, 1024);
#pragma unroll
                        for (int c = 2 * c2; c < 2 * c2 + 2; c++) {
                            const uint64_t vd =
                                sdesc(base + L::K_OFF + 2 * c * K_CHUNK + kk * 2048, K_CHUNK, 1024);
                            mma_bf16(tmem + 2 * HPC * c, vd, pd, id_o, kk > 0);
                        }
                    }
                    mma_commit(c2 == 0 ? bar_pv : bar);
                }
            }
            if (ok) ok = warp < 4 ? mbar_wait_bounded(bar_pv, pv_phase, WAIT_NS) : mbar_wait_bounded(bar, 1, WAIT_NS);
            if (pv_issued) pv_phase ^= 1;
            tc_fence_after();

            // ---- publish this CTA's unnormalized O, row maxima and sums in the
            // cluster's exchange slot (L2), laid out [source][64-channel slice][HPC
            // heads][64 channels]. TMEM lane = channel, so every warp store of one
            // head writes 32 consecutive channels (128 bytes); warps w and w + 4
            // take channel blocks 0-1 and 2-3.
            {
                const int q4 = warp & 3;
                const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
#pragma unroll 1
                for (int c = 2 * (warp >> 2); c < 2 * (warp >> 2) + 2; c++) {
                    const int ch = 128 * c + 32 * q4 + lane;  // this thread's channel
                    float *dst = xo + ((int64_t)rank * CL + (ch >> 6)) * (HPC * 64) + (ch & 63);
                    float v[HPC], vlo[HPC];
                    load_ot<HPC>(lane_addr + 2 * HPC * c, v);
                    load_ot<HPC>(lane_addr + 2 * HPC * c + HPC, vlo);
#pragma unroll
                    for (int i = 0; i < HPC; i++) dst[i * 64] = ok ? v[i] + vlo[i] : 0.0f;
                }
                if (warp < HPC / 16 && half == 0) {
                    xm[rank * HPC + h] = ok ? m_s[h] : -INFINITY;
                    xl[rank * HPC + h] = ok ? l_s[h] : 0.0f;
                }
            }
            __syncthreads();
            // the cluster barrier's release/acquire orders these stores for the
            // cluster's CTAs, the only readers of the slot
            tc_fence_before();
            cluster_sync();  // all partial results of this item are in the slot

            // ---- combine: this CTA owns channels [64 rank, 64 rank + 64); the
            // slice of source r is contiguous at xo[r][rank]. Thread t takes the
            // 16-byte chunks e = 4 (t + 256 u), u < HPC / 16, of the [HPC heads][64
            // channels] slice.
            float *out = lay.out[l];
            {
                constexpr int U = HPC / 16;
                float *wts = reinterpret_cast<float *>(sm + L::P_OFF);  // [HPC heads][8] weight / den
                if (tid < HPC) {
                    float mr[CL], lr[CL];
#pragma unroll
                    for (int r = 0; r < CL; r++) {
                        mr[r] = __ldcg(xm + r * HPC + tid);
                        lr[r] = __ldcg(xl + r * HPC + tid);
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
                float4 f[U][CL];
#pragma unroll
                for (int u = 0; u < U; u++)
#pragma unroll
                    for (int r = 0; r < CL; r++)
                        f[u][r] = __ldcg(reinterpret_cast<const float4 *>(
                                             xo + ((int64_t)r * CL + rank) * (HPC * 64)) +
                                         tid + 256 * u);
                __syncthreads();  // weights ready
#pragma unroll
                for (int u = 0; u < U; u++) {
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
                    *reinterpret_cast<float4 *>(out + (bq * HQ + hg * HPC + hh) * (int64_t)CH +
                                                (int)rank * 64 + ch) = acc;
                }
            }
            // this CTA's part of the row's layer-l output is written
            if (NL > 1 && !row_major) {
                __syncthreads();  // every thread's output stores precede the release below
                if (tid == 0) red_release_gpu_add(lay.row_done + bq, 1);
            }
            // The slot, the tiles and TMEM are free for the next item once every
            // CTA of the cluster has combined. With keep and several clusters per
            // row, the next use is the next layer of the same row, which first
            // waits until every CTA of the row has written this layer's output
            // (after its combine); after the last item of the last layer nothing
            // is shared any more.
            const bool last = step == n_mine * NL - 1;
            if ((!keep || row_major) && !last) cluster_sync();
        }
    }
    if (!ok) {
        atomicExch(&g_attn_error, 1);
        if (a.err) atomicExch(a.err, 1);
    }
    // copies still in flight into this CTA's shared memory land before it exits
    if (tid == 0 && ld_pending) (void)mbar_wait_bounded(bar_ld, ld_phase, WAIT_NS);
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace tc

// Heads per CTA for a call of `rows` query rows and one layer: split the 64
// heads while the (row, head group) items still run in one wave of 8-CTA
// clusters (15 fit on a B200 at one CTA per SM). Per-phase timestamps at 200K
// context put a 1-row call at 10.7 / 11.1 / 12.4 us from first CTA start to
// last CTA end with 16 / 32 / 64 heads per CTA, a 6-row call at 12.0 us with 32
// and 13.3 us with 64. With dependent launches two consecutive layers share
// the 15 cluster slots: a layer that gathers before its wait (prefetch) keeps
// to 7 clusters and one that waits first to 8, so that the next layer's
// clusters all start (and gather) while this one runs.
static int tc_heads_per_cta(int64_t rows, bool pdl, bool prefetch) {
    if (!pdl) return rows <= 2 ? 16 : rows <= 7 ? 32 : 64;
    const int64_t lim = prefetch ? 7 : 8;
    return 4 * rows <= lim ? 16 : 2 * rows <= lim ? 32 : 64;
}

// Clusters of the HPC-head kernel that can be resident at once (the
// persistent loop then runs in one wave); MAX_CLUSTERS if the query fails.
template <int HPC>
int tc_max_active_clusters() {
    static PerDevice cache;
    return cache.get([] {
        int n = 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(tc::CL, tc::MAX_CLUSTERS, 1);
        cfg.blockDim = dim3(tc::THREADS, 1, 1);
        cfg.dynamicSmemBytes = tc::Cfg<HPC>::SMEM_BYTES;
        cudaLaunchAttribute at;
        at.id = cudaLaunchAttributeClusterDimension;
        at.val.clusterDim.x = tc::CL;
        at.val.clusterDim.y = 1;
        at.val.clusterDim.z = 1;
        cfg.attrs = &at;
        cfg.numAttrs = 1;
        int m = 0;
        if (cudaFuncSetAttribute(tc::attn_tc_kernel<HPC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc::Cfg<HPC>::SMEM_BYTES) == cudaSuccess &&
            cudaOccupancyMaxActiveClusters(&m, tc::attn_tc_kernel<HPC>, &cfg) == cudaSuccess && m > 0)
            n = m;
        else
            n = tc::MAX_CLUSTERS;
        (void)cudaGetLastError();
        return n;
    });
}

// Heads per CTA for a launch of a whole layer group: the launch has the GPU to
// itself (no other attention layer runs beside it), so the heads are split as
// finely as the (row, head group) items still fit in one resident wave.
static int tc_group_heads(int64_t rows) {
    if (4 * rows <= tc::MAX_CLUSTERS && 4 * rows <= tc_max_active_clusters<16>()) return 16;
    if (2 * rows <= tc::MAX_CLUSTERS && 2 * rows <= tc_max_active_clusters<32>()) return 32;
    return 64;
}

// Slots per CTA: ks for selected keys, wsz for window rows, each rounded up to
// a multiple of 8 (window boxes then land on 1024-byte boundaries of the tile).
struct TcSplit {
    int ks, wsz;
};
static TcSplit tc_split(const AttnArgs &a) {
    int nwin = a.n_win < a.swa_rows ? a.n_win : a.swa_rows;
    if (a.swa == nullptr || nwin < 0) nwin = 0;
    const int ks = ((a.K + tc::CL - 1) / tc::CL + 7) / 8 * 8;
    const int wsz = ((nwin + tc::CL - 1) / tc::CL + 7) / 8 * 8;
    return {ks, wsz};
}

bool attn_tc_supported(const AttnArgs &a) {
    const int nwin = a.n_win < a.swa_rows ? a.n_win : a.swa_rows;
    const bool has_win = nwin > 0 && a.swa != nullptr;
    const TcSplit sp = tc_split(a);
    return a.C == tc::CH && a.Hq == tc::HQ && a.K > 0 && a.K <= tc::KEYS_MAX &&
           sp.ks + sp.wsz <= tc::T && aligned(a.q, 16) && aligned(a.kv_fp4, 16) &&
           aligned(a.kv_sf, 16) &&
           (!has_win || (aligned(a.swa, 16) && (int64_t)a.B * a.swa_rows >= tc::SWA_BOX)) &&
           (int64_t)a.B * a.Nq * tc::HQ < INT32_MAX && (int64_t)a.B * a.swa_rows < INT32_MAX;
}

// One launch over the layers q[i] / swa[i] / out[i], i < n, that share a's
// selected rows (a.q, a.swa, a.out are layer 0's). row_done: per-row counters
// at row_base (unused when n == 1); *adds receives what the launch adds to
// each of them.
template <int HPC>
static int launch_tc(const AttnArgs &a, const void *const *q, const void *const *swa,
                     float *const *out, int n, int *row_done, int row_base, int *adds,
                     cudaStream_t s) {
    using L = tc::Cfg<HPC>;
    static PerDevice smem_set;
    if (!set_smem_limit_once(smem_set, tc::attn_tc_kernel<HPC>, L::SMEM_BYTES)) return CSA2_ERR_CUDA;
    const int64_t rows = (int64_t)a.B * a.Nq;
    const int64_t items = rows * L::HG;
    const bool has_win = a.swa != nullptr && a.swa_rows > 0 && a.n_win > 0;
    tc::TcLayers lay;
    memset(&lay, 0, sizeof lay);
    lay.n = n;
    lay.row_done = row_done;
    lay.row_base = row_base;
    // clusters that own whole rows follow their layers through the cluster
    // barrier and leave the per-row counters alone
    if (adds) *adds = (n > 1 && L::HG > 1) ? n * L::HG * tc::CL : 0;
    for (int i = 0; i < n; i++) {
        lay.q[i] = q[i];
        lay.swa[i] = swa[i];
        lay.out[i] = out[i];
        if (!make_tmap_2d(&lay.tq[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q[i], tc::CH,
                          (uint64_t)rows * tc::HQ, tc::CH * 2, 64, HPC))
            return CSA2_ERR_CUDA;
        // without a window the map is never used; describe the Q tensor instead
        if (!make_tmap_2d(&lay.tswa[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, has_win ? swa[i] : q[i],
                          tc::CH, has_win ? (uint64_t)a.B * a.swa_rows : (uint64_t)rows * tc::HQ,
                          tc::CH * 2, 64, tc::SWA_BOX))
            return CSA2_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    int64_t clusters = items < tc::MAX_CLUSTERS ? items : tc::MAX_CLUSTERS;
    if (clusters > tc_max_active_clusters<HPC>()) clusters = tc_max_active_clusters<HPC>();
    cfg.gridDim = dim3(tc::CL, (unsigned)clusters, 1);
    cfg.blockDim = dim3(tc::THREADS, 1, 1);
    cfg.dynamicSmemBytes = L::SMEM_BYTES;
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
    const TcSplit sp = tc_split(a);
    if (cudaLaunchKernelEx(&cfg, tc::attn_tc_kernel<HPC>, lay, a, sp.ks, sp.wsz) != cudaSuccess)
        return CSA2_ERR_CUDA;
    return launch_status();
}

static int launch_tc_heads(int hpc, const AttnArgs &a, const void *const *q, const void *const *swa,
                           float *const *out, int n, int *row_done, int row_base, int *adds,
                           cudaStream_t s) {
    switch (hpc) {
    case 16: return launch_tc<16>(a, q, swa, out, n, row_done, row_base, adds, s);
    case 32: return launch_tc<32>(a, q, swa, out, n, row_done, row_base, adds, s);
    default: return launch_tc<64>(a, q, swa, out, n, row_done, row_base, adds, s);
    }
}

int launch_attn_tc(const AttnArgs &a, cudaStream_t s) {
    if (a.ws == nullptr) return CSA2_ERR_WORKSPACE;
    const void *q[1] = {a.q};
    const void *swa[1] = {a.swa};
    float *out[1] = {a.out};
    return launch_tc_heads(tc_heads_per_cta((int64_t)a.B * a.Nq, a.pdl, a.prefetch), a, q, swa, out, 1,
                           nullptr, 0, nullptr, s);
}

int launch_attn_tc_group(const AttnArgs &a, const void *const *q, const void *const *swa,
                         float *const *out, int n, int *row_done, int row_base, int *adds,
                         cudaStream_t s) {
    if (a.ws == nullptr) return CSA2_ERR_WORKSPACE;
    if (n < 1 || n > tc::MAXL || (n > 1 && row_done == nullptr)) return CSA2_ERR_SHAPE;
    for (int i = 0; i < n; i++) {
        if (!q[i] || !out[i] || (a.swa && !swa[i])) return CSA2_ERR_NULL;
        if (!aligned(q[i], 16) || (a.swa && !aligned(swa[i], 16))) return CSA2_ERR_ALIGN;
    }
    return launch_tc_heads(tc_group_heads((int64_t)a.B * a.Nq), a, q, swa, out, n, row_done, row_base,
                           adds, s);
}

int attn_tc_wait_flag(bool clear) { return read_device_flag(tc::g_attn_error, clear); }

size_t attn_tc_workspace_bytes(int B, int Nq) {
    // the largest of the head splits a call of this size can take (any of 16,
    // 32 or 64 heads per cluster, at most MAX_CLUSTERS clusters)
    const int64_t rows = (int64_t)B * Nq;
    size_t most = 0;
    for (int hpc = 16; hpc <= 64; hpc *= 2) {
        const int64_t items = rows * (tc::HQ / hpc);
        const int64_t clusters = items < tc::MAX_CLUSTERS ? items : tc::MAX_CLUSTERS;
        const int64_t slot = (int64_t)tc::CL * hpc * tc::CH + 2 * tc::CL * hpc;
        const size_t bytes = (size_t)clusters * slot * sizeof(float);
        if (bytes > most) most = bytes;
    }
    return most;
}

int attn_group_max_layers() { return tc::MAXL; }

}  // namespace csa2

extern "C" int csa2_attn_resident_clusters(int heads_per_cluster) {
    using namespace csa2;
    switch (heads_per_cluster) {
    case 16: return tc_max_active_clusters<16>();
    case 32: return tc_max_active_clusters<32>();
    case 64: return tc_max_active_clusters<64>();
    default: return CSA2_ERR_RANGE;
    }
}
