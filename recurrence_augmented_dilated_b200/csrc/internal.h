// internal.h -- declarations shared between the C ABI layer and the kernels (not installed).
#pragma once

#include <atomic>
#include <stddef.h>
#include <stdint.h>

#include "../../include/rat.h"

namespace rat {

// Every device-side wait gives up after this long and records RAT_ERR_TIMEOUT.
constexpr uint64_t kWaitLimitNs = 2000ull * 1000ull * 1000ull;   // 2 s

// First 256 bytes of every workspace.
struct WsHeader {
    int error;          // first device-side error of any launch since the last rat_sync_status
    uint32_t detail;    // where it happened (kernel-specific code)
    uint32_t epoch;     // launch counter: tags look-back flags so they never need clearing
    uint32_t ticket;    // CTA ticket dispenser (reset by the last CTA of each launch)
    uint32_t done;      // CTAs finished in the current launch
    uint32_t pad[59];
};
static_assert(sizeof(WsHeader) == 256, "workspace header must be 256 bytes");

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------------------- recurrence
struct RecurParams {
    const void *k, *v, *a;
    const float *h0k, *h0v;
    void *yk, *yv;
    float *hTk, *hTv;
    int BH, T, d, nchunks;
    long long pos0;
    int rope;                   // 1: rotate k~
    WsHeader *hdr;
    // look-back records, one 64-bit word per value: (launch tag << 32) | float bits, so every
    // value validates itself and needs no separate flag or fence
    uint64_t *agg;              // [BH * nchunks][3][d]   A, Bk, Bv of the chunk
    uint64_t *pre;              // [BH * nchunks][2][d]   inclusive state Hk, Hv after the chunk
    int rope_f32;               // positions small enough for float32 angles (pos0 + T <= 2^13)
    float theta_f[64];
    double theta[64];           // RoPE frequency theta_c = base^(-2c/d), c < d/2
    float step_cos[64], step_sin[64];   // cos/sin(theta_c): one-position rotation
    long long fault_chunk;      // test hook: chunk index that never publishes (-1: none)
    unsigned long long wait_ns; // bound of each look-back wait
    long long reset;            // > 0: state zeroed before every position that is a multiple (chunk-local recurrence)
};
// fixed-window recurrence: each state restarted kWindowRows positions back
constexpr int kWindowRows = 64;
struct WindowParams {
    const void *k, *v, *a;
    const void *pk, *pv, *pa;   // [BH][kWindowRows][d] positions before row 0, or all null
    void *yk, *yv;
    int BH, T, d, nblk;         // nblk = ceil(T / kWindowRows)
    long long pos0;
    int rope, rope_f32;
    WsHeader *hdr;
    float theta_f[64];
    double theta[64];
    float step_cos[64], step_sin[64];
};
int launch_window(const WindowParams &p, int dtype, void *stream);

// backward of the fixed-window recurrence (one launch, no waits between CTAs)
struct WindowBwdParams {
    const void *k, *v, *a;          // forward inputs
    const void *pk, *pv, *pa;       // [BH][kWindowRows][d] history rows, or all null
    const void *dyk, *dyv;          // upstream gradients of k~, v~
    void *dk, *dv, *da;             // outputs
    void *dpk, *dpv, *dpa;          // gradients of the history rows, or all null
    int BH, T, d, nblk;             // nblk = ceil(T / kWindowRows)
    long long pos0;
    int rope, rope_f32;
    float theta_f[64];
    double theta[64];
    float step_cos[64], step_sin[64];
    float step64_cos[64], step64_sin[64];   // rotation by kWindowRows positions
};
int launch_window_bwd(const WindowBwdParams &p, int dtype, void *stream);

// backward of the recurrence step (reduce, carry and output launches over 64-row chunks)
struct RecurBwdParams {
    const void *k, *v, *a;          // forward inputs
    const void *yk, *yv;            // forward outputs k~ (rotated), v~
    const void *dyk, *dyv;          // upstream gradients of k~, v~
    const float *h0k, *h0v;         // initial state, or null
    const float *dhTk, *dhTv;       // gradient of the final state, or null
    void *dk, *dv, *da;             // outputs
    float *dh0k, *dh0v;             // gradient of the initial state, or null
    WsHeader *hdr;
    // look-back records, one 64-bit word per value: (launch tag << 32) | float bits
    uint64_t *agg;                  // [BH * nch][3][d]  map (A, Bk, Bv) of each chunk
    uint64_t *pre;                  // [BH * nch][2][d]  carry leaving each chunk to the left
    int BH, T, d, nch;
    long long pos0;
    int rope, rope_f32;
    float theta_f[64];
    double theta[64];
    float step_cos[64], step_sin[64];
    long long reset;                // > 0: the chunk-local form (state restarted at multiples)
    long long fault_chunk;          // test hook: chunk index that never publishes (-1: none)
    unsigned long long wait_ns;     // bound of each look-back wait
};
int recur_bwd_chunk_rows(int d, int dtype);
size_t recur_bwd_workspace_bytes(int BH, int T, int d);
int launch_recur_bwd(const RecurBwdParams &p, int dtype, void *stream);

int recur_chunk_rows(int d, int dtype);
size_t recur_workspace_bytes(int BH, int T, int d, int dtype);
int launch_recur(const RecurParams &p, int dtype, void *stream);

// ---------------------------------------------------------------------------- attention
constexpr int kMaxHeads = 256;

struct AttnSimtParams {
    const void *q, *k, *v;
    void *o;
    int B, H, T, d, W;
    long long pos0;
    int rope;
    float scale_log2;           // softmax scale * log2(e)
    int n_sink;                 // attention sinks: the first n_sink positions join every key set
    int top_k;                  // chunks (scored by their chunk-end keys) attended in full, <= 16
    float *lse;                 // [B*H][T] or null: log2 of each row's softmax denominator
    int Dh[kMaxHeads];
    double theta[64];
};
int launch_attn_simt(const AttnSimtParams &p, int dtype, void *stream);

struct AttnSm100Args {
    const void *q, *k, *v;
    void *o;
    int B, H, T, d, W;
    long long pos0;
    int rope;
    float scale_log2;
    const int32_t *Dh;          // host [H]
    int n_sink;                 // attention sinks; the caller ensures n_sink < D (D > 1) and <= 64
    int top_k;                  // > 0: top-k chunk selection (then n_sink == 0, T <= 65536)
    float *lse;                 // [B*H][T] or null: log2 of each row's softmax denominator
    double theta[64];
};
int launch_attn_sm100(const AttnSm100Args &a, void *stream);

// Opt kernel `fn` into `bytes` of dynamic shared memory on the current device, once per device
// (bit `dev` of *done_mask records it; the mask is atomic, so concurrent host threads may call
// this -- at worst two of them both set the attribute).  Returns a rat_status.
inline int set_smem_attr(const void *fn, uint32_t bytes, std::atomic<uint64_t> *done_mask) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RAT_ERR_CUDA;
    if (done_mask->load(std::memory_order_acquire) >> dev & 1) return RAT_OK;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return RAT_ERR_CUDA;
    done_mask->fetch_or(1ull << dev, std::memory_order_release);
    return RAT_OK;
}

// Number of SMs of the current device (0 on error).
inline int current_sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return sms;
}
int attn_error_word(void *stream, bool clear);
unsigned attn_error_where();
unsigned attn_error_waiting();
extern int g_attn_block_keys;

// ---------------------------------------------------------------------------- cache / decode
struct CompressParams {
    const void *k, *v;
    const float *hTk, *hTv;
    void *kdil, *vdil, *kwin, *vwin;
    float *hk, *hv;
    int B, H, T, d, W, Tcap, esize;
    long long pos0;
    long long total_cap;
    int Dh[kMaxHeads];
    long long off[kMaxHeads];
    int blk0[kMaxHeads + 1];    // filled by launch_compress: first CTA of head h within a batch row
    // paged cache (page_table non-null): the input holds one sequence (B = 1), stored as
    // sequence `seq` of the cache; dil entry i of head h goes to pool row
    // page_table[seq * H + h][i >> page_shift] * page_entries + (i & (page_entries - 1))
    const int32_t *page_table;
    int page_shift, max_pages, n_pages, seq;
    long long *seq_pos;         // [B] set to pos0 + T for sequence seq
    WsHeader *hdr;              // receives RAT_ERR_INVALID for a page index outside the pool
    void *ksink, *vsink;        // [B][H][n_sink][d]: positions below n_sink (attention sinks)
    int n_sink;
};
int launch_compress(const CompressParams &p, void *stream);

// backward of the dilated attention (CUDA cores, float32 accumulation)
struct AttnBwdParams {
    const void *q, *k, *v, *o, *dO;
    void *dq, *dk, *dv;
    void *qh;                   // workspace [B*H][T][d] of dtype: RoPE(q) as the attention uses it
    float *lse;                 // [B*H][T]: log2 of each query's softmax denominator (workspace,
                                // or the forward's output when lse_given)
    int lse_given;              // 1: lse holds the forward's values, the dq launch skips its pass 1
    float *delta;               // workspace [B*H][T]: <dO_t, o_t>
    int B, H, T, d, W, n_sink;
    long long pos0;
    int rope;
    float scale, scale_log2;
    int Dh[kMaxHeads];
    double theta[64];
    WsHeader *hdr;              // workspace header: device-side errors of the tensor-core kernels
};
size_t attn_bwd_workspace_bytes(int B, int H, int T, int d, int dtype);
int launch_attn_bwd(const AttnBwdParams &p, int dtype, void *stream);
// tensor-core form (bf16, d = 128, no sinks, at most four dilations > 1 in a launch)
bool attn_bwd_sm100_supported(const AttnBwdParams &p, int dtype);
int launch_attn_bwd_sm100(const AttnBwdParams &p, void *stream);

struct DecodeParams {
    const void *q, *k, *v, *a;
    void *o;
    int window_rec;             // > 0: the fixed-window recurrence over raw rings of window_rec rows
    void *kraw, *vraw, *araw;   // [B*H][window_rec][d] raw k, v, gate logits, slot p mod window_rec
    void *kdil, *vdil, *kwin, *vwin;
    float *hk, *hv;
    int B, H, d, W, Tcap, splits;
    long long t;                // position of the new token
    long long reset;            // > 0: state dropped before every position that is a multiple
    long long total_cap;
    int rope;
    float scale_log2;
    WsHeader *hdr;
    uint32_t *tickets;          // [B*H]
    float *part_ml;             // [B*H][splits][2]  running max (log2 units) and sum
    float *part_o;              // [B*H][splits][d]
    int Dh[kMaxHeads];
    long long off[kMaxHeads];
    double theta[64];
    // paged cache with per-sequence positions (launch_decode with paged = true): kdil / vdil are
    // the page pools, entry i of slice (b, h) is row page_table[bh][i >> page_shift] *
    // page_entries + (i & (page_entries - 1)) of the pool
    long long *seq_pos;         // [B] position of sequence b's new token; advanced by the kernel
    uint32_t *seq_ticket;       // [B] CTAs of sequence b finished (the last one advances seq_pos)
    const int32_t *page_table;  // [B * H][max_pages]
    int page_shift, max_pages, n_pages;
    void *ksink, *vsink;        // [B * H][n_sink][d]: positions 0 .. n_sink-1 (attention sinks)
    int n_sink;
};
int decode_splits(int B, int H, int Tcap, const int32_t *Dh, int W);
int decode_splits_for_keys(int B, int H, long long max_keys);
size_t decode_workspace_bytes(int B, int H, int d, int splits);
int launch_decode(const DecodeParams &p, int dtype, void *stream, bool paged = false);

}  // namespace rat
