// Shared definitions of the sparse-attention kernels.
#pragma once

#include "common.cuh"

namespace csa2 {

struct AttnArgs {
    const void *q;         // bf16 [B][Nq][Hq][C]
    const uint8_t *kv_fp4; // [B][cap][C/2]
    const uint8_t *kv_sf;  // [B][cap][C/16]
    int64_t cap;
    const int32_t *topk;   // [B][Nq][K]
    int K;
    const void *swa;       // bf16 [B][swa_rows][C]
    const int64_t *swa_pos0;
    int swa_rows;
    const int64_t *q_pos;  // [B][Nq] or NULL
    int n_win;
    int B, Nq, Hq, C;
    float scale;
    float *out;            // fp32 [B][Nq][Hq][C]
    void *ws;
    // Launch with programmatic stream serialization (the kernel may start
    // while the previous kernel on the stream runs; it waits for that grid
    // before reading Q or the window rows and before writing anything).
    bool pdl;
    // With pdl: topk, kv_fp4/kv_sf and swa_pos0 were written two or more
    // kernels earlier, so the selected rows may be gathered and dequantized
    // before the wait.
    bool prefetch;
    // Scales of the FP4 rows: E4M3 per 16 channels (kv_sf [B][cap][C/16]), or
    // with mx the MXFP4 variant's E8M0 per 32 channels (kv_sf [B][cap][C/32]).
    bool mx;
    // The call's error word (the first word of the caller's workspace), or
    // NULL: a kernel that gives up a bounded wait sets it to 1 besides the
    // library's device flag.
    int *err = nullptr;
};

// Bytes at the start of a workspace that hold the call's error word.
constexpr size_t kErrWordBytes = 256;

// Sliding-window rows of query bq: rows [row0, row0 + n) of the SWA tensor,
// i.e. positions max(0, p - n_win + 1) .. p that the tensor holds.
struct AttnWindow {
    int64_t row0;
    int n;
};

__device__ __forceinline__ AttnWindow attn_window(const AttnArgs &a, int b, int64_t bq) {
    AttnWindow w{0, 0};
    if (a.n_win <= 0 || a.swa_rows <= 0 || !a.swa) return w;
    const int64_t pos0 = a.swa_pos0 ? a.swa_pos0[b] : 0;
    const int64_t p = a.q_pos ? a.q_pos[bq] : pos0 + a.swa_rows - 1;
    int64_t lo = p - a.n_win + 1;
    if (lo < 0) lo = 0;
    if (lo < pos0) lo = pos0;
    int64_t hi = p;
    if (hi > pos0 + a.swa_rows - 1) hi = pos0 + a.swa_rows - 1;
    if (hi >= lo) {
        w.row0 = lo - pos0;
        w.n = (int)(hi - lo + 1);
    }
    return w;
}

size_t attn_workspace_bytes(int B, int Nq, int Hq, int C, int K, int n_win);
// The kernels' scratch (AttnArgs::ws) without the error word.
size_t attn_scratch_bytes(int B, int Nq, int Hq, int C, int K);
// A standalone call (csa2_sparse_attn_decode): the error word at the start of
// ws is cleared, then the call is checked and launched with the rest as scratch.
int attn_call(AttnArgs a, size_t ws_bytes, cudaStream_t s);
// Validates the arguments of a sparse-attention call (status codes of
// csa2_sparse_attn_decode) and launches it.
// With validate_only, only the checks run (CSA2_OK when the call would launch).
int attn_checked_launch(const AttnArgs &a, size_t ws_bytes, cudaStream_t s,
                        bool validate_only = false);
int launch_attn(const AttnArgs &a, cudaStream_t s);
int launch_attn_general(const AttnArgs &a, cudaStream_t s);
bool attn_tc_supported(const AttnArgs &a);
size_t attn_tc_workspace_bytes(int B, int Nq);
int launch_attn_tc(const AttnArgs &a, cudaStream_t s);
// The tensor-core kernel over a group of n layers that share a's selected rows
// (layer i: Q q[i], window rows swa[i], output out[i]; a.q / a.swa / a.out are
// ignored). Layer i + 1 of a query row runs once layer i of that row is
// written: row_done holds one counter per query row (B Nq ints, each equal to
// row_base at launch; used when n > 1) and *adds receives how much the launch
// adds to each.
int launch_attn_tc_group(const AttnArgs &a, const void *const *q, const void *const *swa,
                         float *const *out, int n, int *row_done, int row_base, int *adds,
                         cudaStream_t s);
// Most layers one group launch takes (kMaxGroupLayers).
int attn_group_max_layers();
constexpr int kMaxGroupLayers = 8;
// One CTA per query row (attention_rows.cu): no workspace; for calls of
// kAttnRowsMin rows or more (below that the split-key clusters measured
// faster: at 32 rows and fewer, the decode batches).
bool attn_rows_supported(const AttnArgs &a);
int launch_attn_rows(const AttnArgs &a, cudaStream_t s);
constexpr int64_t kAttnRowsMin = 64;

}  // namespace csa2
