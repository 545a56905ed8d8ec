// Library-level entry points: status strings, ABI version and the decode step
// over a CSA2 layer stack.
//
// "DeepSeek-V4.1-Flash: 890 Bytes Per Token, 437x Smaller KV Cache", CSA2
// section: each layer is statically Full, Reindex or Reuse; Full layers build
// the pool and a fresh top-512, Reindex layers rescore the pool with their own
// indexer Q, Reuse layers attend the indices of the nearest Full/Reindex
// layer; every layer attends with its own main Q and SWA KV.
#include "attention.cuh"

using namespace csa2;

extern "C" const char *csa2_status_string(int status) {
    switch (status) {
        case CSA2_OK: return "ok";
        case CSA2_ERR_NULL: return "a required pointer is NULL";
        case CSA2_ERR_SHAPE: return "a size is outside the supported range";
        case CSA2_ERR_ALIGN: return "a pointer or row size breaks the alignment rule";
        case CSA2_ERR_RANGE: return "a host-side value is out of range";
        case CSA2_ERR_WORKSPACE: return "workspace missing or too small";
        case CSA2_ERR_CUDA: return "a CUDA launch failed";
        case CSA2_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait on the device";
        default: return "unknown status";
    }
}

extern "C" int csa2_abi_version(void) { return CSA2_ABI_VERSION; }

extern "C" int csa2_workspace_status(const void *ws, int clear, void *stream) {
    if (!ws) return CSA2_ERR_NULL;
    cudaStream_t s = (cudaStream_t)stream;
    int v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return CSA2_ERR_CUDA;
    if (clear && v && cudaMemsetAsync(const_cast<void *>(ws), 0, sizeof(int), s) != cudaSuccess)
        return CSA2_ERR_CUDA;
    return v ? CSA2_ERR_DEVICE_TIMEOUT : CSA2_OK;
}

namespace {

uint32_t *topk_hist_ptr_of(void *ws) { return static_cast<uint32_t *>(ws); }

constexpr size_t kAlign = 256;
inline size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct StackWs {
    int *err;          // the call's error word (set when a kernel gives up a bounded wait)
    float *tok;
    float *blk;
    int32_t *n_blk;
    float *pscore;
    int32_t *ppos;
    int *row_done;     // per-row layer counters of the grouped attention launches
    void *sel_blk;     // histogram-fed top-k workspace of the pool selection
    void *sel_tok;     // ... and of the token top-512
    size_t hist_bytes; // leading bytes of each that must be zero before a step
    size_t zero_bytes; // bytes from err that must be zero (error word, counters, sel_blk's histogram)
    void *attn;
    size_t attn_bytes;
    size_t total;
};

// Layout: the error word first (where csa2_workspace_status reads it), then
// the regions that start every step at zero (the attention layer counters and
// the pool selection's histogram follow it contiguously, so one memset clears
// all three), then the scores and the attention scratch.
StackWs stack_layout(void *base, int B, int Hq, int C, int64_t cap) {
    StackWs w{};
    size_t off = 0;
    char *p = static_cast<char *>(base);
    const int64_t nblk = (cap + 7) / 8;
    const int64_t P8 = (int64_t)kPoolBlocks * kBlockTokens;
    w.err = reinterpret_cast<int *>(p + off);
    off += kErrWordBytes;
    w.row_done = reinterpret_cast<int *>(p + off);
    off += up(sizeof(int) * (size_t)B);
    w.sel_blk = p + off;
    off += up(topk_hist_ws_bytes(B, kPoolBlocks));
    w.sel_tok = p + off;
    off += up(topk_hist_ws_bytes(B, kTopK));
    w.hist_bytes = topk_hist_zero_bytes(B);
    w.zero_bytes = kErrWordBytes + up(sizeof(int) * (size_t)B) + w.hist_bytes;
    w.tok = reinterpret_cast<float *>(p + off);
    off += up(sizeof(float) * (size_t)B * cap);
    w.blk = reinterpret_cast<float *>(p + off);
    off += up(sizeof(float) * (size_t)B * nblk);
    w.n_blk = reinterpret_cast<int32_t *>(p + off);
    off += up(sizeof(int32_t) * (size_t)B);
    w.pscore = reinterpret_cast<float *>(p + off);
    off += up(sizeof(float) * (size_t)B * P8);
    w.ppos = reinterpret_cast<int32_t *>(p + off);
    off += up(sizeof(int32_t) * (size_t)B * P8);
    w.attn = p + off;
    w.attn_bytes = up(attn_scratch_bytes(B, 1, Hq, C, kTopK));
    off += w.attn_bytes;
    w.total = off;
    return w;
}

}  // namespace

extern "C" size_t csa2_decode_stack_workspace_size(int B, int Hq, int C, int H, int D,
                                                   int64_t cap) {
    (void)H;
    (void)D;
    if (B < 0 || cap < 1) return 0;
    return stack_layout(nullptr, B, Hq, C, cap).total;
}

extern "C" int csa2_decode_stack(const csa2_layer *layers, int n_layers,
                                 const void *kv_new_bf16, const int8_t *k_idx,
                                 const float *k_scale, uint8_t *kv_fp4, uint8_t *kv_sf,
                                 int64_t cap, const int64_t *ctx_len,
                                 const int64_t *swa_pos0, int swa_rows, int B, int Hq, int C,
                                 int H, int D, float softmax_scale, int32_t *pool,
                                 int pool_ready, void *const *scan_events, void *ws,
                                 size_t ws_bytes, void *stream) {
    if (!layers || !k_idx || !k_scale || !kv_fp4 || !kv_sf || !ctx_len || !swa_pos0 || !pool)
        return CSA2_ERR_NULL;
    if (n_layers < 1 || B < 1 || cap < 1 || C < 32 || C % 32) return CSA2_ERR_SHAPE;
    if (kv_new_bf16 && !aligned(kv_new_bf16, 16)) return CSA2_ERR_ALIGN;
    const StackWs w = stack_layout(ws, B, Hq, C, cap);
    if (!ws || ws_bytes < w.total) return CSA2_ERR_WORKSPACE;
    // the kernels read the workspace's histograms, lists and exchange slots
    // with 16-byte accesses
    if (!aligned(ws, 16)) return CSA2_ERR_ALIGN;
    // host-side schedule check before anything is launched
    bool have_pool = pool_ready != 0, have_idx = false;
    for (int l = 0; l < n_layers; l++) {
        const csa2_layer &L = layers[l];
        if (!L.q || !L.out || (swa_rows > 0 && !L.swa)) return CSA2_ERR_NULL;
        if (L.mode == CSA2_MODE_FULL) {
            if (!L.q_idx || !L.topk) return CSA2_ERR_NULL;
            have_pool = have_idx = true;
        } else if (L.mode == CSA2_MODE_REINDEX) {
            if (!L.q_idx || !L.topk) return CSA2_ERR_NULL;
            if (!have_pool) return CSA2_ERR_RANGE;
            have_idx = true;
        } else if (L.mode == CSA2_MODE_REUSE) {
            if (!have_idx) return CSA2_ERR_RANGE;
        } else {
            return CSA2_ERR_RANGE;
        }
    }
    const int64_t nblk = (cap + 7) / 8;
    const int P8 = kPoolBlocks * kBlockTokens;
    const int32_t *cur = nullptr;
    bool scan_timed = false;
    int st;
    cudaStream_t s = (cudaStream_t)stream;
    // The append of the new rows, and the error word, the selection histograms
    // and counters and the attention layer counters set to zero (every
    // finishing top-k kernel also leaves its rows clear for the next
    // producer), in one kernel.
    st = launch_decode_step_begin((const uint16_t *)kv_new_bf16, B, C, ctx_len, cap, kv_fp4, kv_sf,
                                  w.err, w.zero_bytes, w.sel_tok, w.hist_bytes, s);
    if (st) return st;
    uint32_t *hist_blk = topk_hist_ptr_of(w.sel_blk);
    uint32_t *hist_tok = topk_hist_ptr_of(w.sel_tok);
    int row_base = 0;  // value of every per-row layer counter before the next group
    for (int l = 0; l < n_layers;) {
        const csa2_layer &L = layers[l];
        if (L.mode == CSA2_MODE_FULL) {
            const bool timed = scan_events && !scan_timed;
            if (timed) cudaEventRecord((cudaEvent_t)scan_events[0], (cudaStream_t)stream);
            st = launch_index_full_hist(L.q_idx, k_idx, k_scale, ctx_len, B, H, D, cap, w.tok, w.blk,
                                        w.n_blk, hist_blk, s);
            if (st) return st;
            if (timed) {
                cudaEventRecord((cudaEvent_t)scan_events[1], (cudaStream_t)stream);
                scan_timed = true;
            }
            // the pool and the top-512 among the pooled tokens in one selection
            // (a compaction kernel first for rows of more than 65,536 blocks)
            st = launch_pool_and_tokens(w.blk, w.n_blk, B, nblk, kPoolBlocks, pool, w.sel_blk, w.tok,
                                        ctx_len, cap, kTopK, L.topk, s);
            if (st) return st;
            cur = L.topk;
        } else if (L.mode == CSA2_MODE_REINDEX) {
            // timed when the stack has no Full layer before it
            const bool timed = scan_events && !scan_timed;
            if (timed) cudaEventRecord((cudaEvent_t)scan_events[0], (cudaStream_t)stream);
            st = launch_reindex_hist(L.q_idx, k_idx, k_scale, pool, ctx_len, B, H, D, cap,
                                     kPoolBlocks, w.pscore, w.ppos, hist_tok, s);
            if (st) return st;
            if (timed) {
                cudaEventRecord((cudaEvent_t)scan_events[1], (cudaStream_t)stream);
                scan_timed = true;
            }
            st = launch_topk_from_hist(w.pscore, w.ppos, nullptr, B, P8, kTopK, L.topk, w.sel_tok,
                                       s);
            if (st) return st;
            cur = L.topk;
        }
        // The attention group: this layer and the Reuse layers after it, which
        // attend the same selected rows. Every kernel of the step is launched
        // with programmatic stream serialization.
        int g = 1;
        while (l + g < n_layers && g < attn_group_max_layers() &&
               layers[l + g].mode == CSA2_MODE_REUSE)
            g++;
        // A launch led by a Reuse layer (a run of Reuse layers longer than one
        // launch takes, or layers launched one by one) follows an attention
        // launch, and its indices come from an earlier selection kernel, so it
        // gathers and dequantizes its rows before waiting; Q and the window rows
        // (the layers' own inputs) are read after the wait.
        AttnArgs aa{L.q, kv_fp4, kv_sf, cap, cur, kTopK, L.swa, swa_pos0, swa_rows, nullptr,
                    CSA2_N_WIN, B, 1, Hq, C, softmax_scale, L.out, w.attn, true,
                    L.mode == CSA2_MODE_REUSE, false, w.err};
        st = attn_checked_launch(aa, w.attn_bytes, s, /*validate_only=*/true);
        if (st) return st;
        if (attn_tc_supported(aa) && (int64_t)B < kAttnRowsMin) {
            // one launch for the group; layer i + 1 of a sequence follows layer i
            // of that sequence through the per-row counters
            const void *gq[kMaxGroupLayers], *gswa[kMaxGroupLayers];
            float *gout[kMaxGroupLayers];
            for (int i = 0; i < g; i++) {
                gq[i] = layers[l + i].q;
                gswa[i] = layers[l + i].swa;
                gout[i] = layers[l + i].out;
            }
            int adds = 0;
            st = launch_attn_tc_group(aa, gq, gswa, gout, g, w.row_done, row_base, &adds, s);
            if (st) return st;
            row_base += adds;
        } else {
            for (int i = 0; i < g; i++) {
                const csa2_layer &Li = layers[l + i];
                aa.q = Li.q;
                aa.swa = Li.swa;
                aa.out = Li.out;
                aa.prefetch = i > 0 || L.mode == CSA2_MODE_REUSE;
                st = attn_checked_launch(aa, w.attn_bytes, s);
                if (st) return st;
            }
        }
        l += g;
    }
    return CSA2_OK;
}
