// rat_abi.cu -- the C ABI: argument validation, workspace carving and kernel dispatch.
//
// Every entry point validates on the host and returns a rat_status synchronously; all GPU
// work is enqueued on the caller's stream.  No entry point allocates device memory.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "internal.h"

using namespace rat;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool supported_d(int d) { return d == 64 || d == 128; }
bool valid_dtype(int dt) { return dt == RAT_F32 || dt == RAT_BF16; }
int esize(int dt) { return dt == RAT_F32 ? 4 : 2; }

// theta_c = base^(-2c/d), c < d/2 (RoFormer frequencies), in float64.
void rope_theta(double base, int d, double *theta) {
    for (int c = 0; c < d / 2; ++c) theta[c] = std::pow(base, -2.0 * (double)c / (double)d);
    for (int c = d / 2; c < 64; ++c) theta[c] = 0.0;
}

long long total_capacity(int H, int Tcap, const int32_t *Dh, long long *off) {
    long long total = 0;
    for (int h = 0; h < H; ++h) {
        if (off) off[h] = total;
        total += Tcap / Dh[h];
    }
    return total;
}

bool valid_cache(const rat_kv_cache *c) {
    if (!c || c->B < 1 || c->H < 1 || c->H > kMaxHeads || !supported_d(c->d) || c->W < 0 ||
        c->Tcap < 1 || !valid_dtype(c->dtype) || !c->D || c->reset_every < 0 || c->n_sink < 0)
        return false;
    // the fixed-window form (L* = 64) has no chunk-local restarts
    if (c->window_rec != 0 && c->window_rec != kWindowRows) return false;
    if (c->window_rec > 0 && c->reset_every != 0) return false;
    for (int h = 0; h < c->H; ++h)
        if (c->D[h] < 1) return false;
    return true;
}

// the raw rings of a cache with window_rec > 0 (none needed otherwise)
bool raw_rings_ok(const rat_kv_cache *c) {
    return c->window_rec == 0 || (c->k_raw && c->v_raw && c->a_raw && aligned16(c->k_raw) &&
                                  aligned16(c->v_raw) && aligned16(c->a_raw));
}

bool valid_paged_cache(const rat_paged_kv_cache *c) {
    if (!c || c->B < 1 || c->H < 1 || c->H > kMaxHeads || !supported_d(c->d) || c->W < 0 ||
        !valid_dtype(c->dtype) || !c->D || c->reset_every < 0 || c->page_entries < 1 ||
        (c->page_entries & (c->page_entries - 1)) != 0 || c->max_pages < 1 || c->n_pages < 1)
        return false;
    if ((long long)c->max_pages * c->page_entries > (1ll << 40)) return false;
    for (int h = 0; h < c->H; ++h)
        if (c->D[h] < 1) return false;
    if (!c->k_pool || !c->v_pool || !c->page_table || !c->h_k || !c->h_v || !c->pos) return false;
    if (!aligned16(c->k_pool) || !aligned16(c->v_pool)) return false;
    if (c->W > 0 && (!c->k_win || !c->v_win || !aligned16(c->k_win) || !aligned16(c->v_win)))
        return false;
    return true;
}

int log2_exact(int x) {
    int s = 0;
    while ((1 << s) < x) ++s;
    return s;
}

// Test hook state: armed by rat_debug_inject_lookback_fault, consumed by the next
// rat_recur_prefill issued from the same host thread.
thread_local long long g_fault_chunk = -1;
thread_local unsigned long long g_fault_wait_ns = 0;

}  // namespace

extern "C" {

int rat_debug_inject_lookback_fault(int64_t chunk, int64_t wait_limit_ns) {
    if (chunk < 1 || wait_limit_ns < 1000000 || wait_limit_ns > (int64_t)kWaitLimitNs)
        return RAT_ERR_INVALID;
    g_fault_chunk = chunk;
    g_fault_wait_ns = (unsigned long long)wait_limit_ns;
    return RAT_OK;
}

const char *rat_status_string(int status) {
    switch (status) {
        case RAT_OK: return "RAT_OK";
        case RAT_ERR_INVALID: return "RAT_ERR_INVALID: invalid argument";
        case RAT_ERR_UNSUPPORTED: return "RAT_ERR_UNSUPPORTED: unsupported configuration";
        case RAT_ERR_CUDA: return "RAT_ERR_CUDA: CUDA call or launch failed";
        case RAT_ERR_TIMEOUT: return "RAT_ERR_TIMEOUT: a bounded device-side wait ran out";
        case RAT_ERR_WORKSPACE: return "RAT_ERR_WORKSPACE: workspace missing or too small";
        default: return "unknown rat_status";
    }
}

const char *rat_version(void) { return "rat-b200 0.1 sm_100a"; }

int64_t rat_attended_keys(int64_t t, int D, int W) {
    if (t < 0 || D < 1) return 0;
    const int64_t We = W > 1 ? W : 1;
    const int64_t win = We < t + 1 ? We : t + 1;
    const int64_t older = t - We + 1;
    return win + (older > 0 ? older / D : 0);
}

int rat_workspace_init(void *ws, size_t ws_bytes, void *stream) {
    if (!ws || ws_bytes < sizeof(WsHeader)) return RAT_ERR_WORKSPACE;
    return cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? RAT_OK : RAT_ERR_CUDA;
}

int rat_sync_status(void *ws, void *stream) {
    if (!ws) return RAT_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return RAT_ERR_CUDA;
    int err = 0;
    WsHeader *hdr = static_cast<WsHeader *>(ws);
    if (cudaMemcpy(&err, &hdr->error, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return RAT_ERR_CUDA;
    if (err != 0) {
        const int zero = 0;
        if (cudaMemcpy(&hdr->error, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return RAT_ERR_CUDA;
    }
    return err;
}

// ------------------------------------------------------------------------------ recurrence
size_t rat_recur_workspace_bytes(int B, int H, int T, int d, int dtype) {
    if (B < 1 || H < 1 || T < 0 || !supported_d(d) || !valid_dtype(dtype)) return 0;
    return recur_workspace_bytes(B * H, T, d, dtype);
}

}  // extern "C"

namespace {
// Both recurrence entry points: reset_every = 0 is the full-sequence recurrence, L > 0 drops
// the state before every absolute position that is a multiple of L.
int recur_prefill(const void *k, const void *v, const void *gate_logit, const float *h0_k,
                  const float *h0_v, void *k_rec, void *v_rec, float *hT_k, float *hT_v, int B,
                  int H, int T, int d, int dtype, int64_t pos0, int64_t reset_every,
                  float rope_base, void *ws, size_t ws_bytes, void *stream) {
    if (B < 1 || H < 1 || T < 0 || !valid_dtype(dtype) || reset_every < 0) return RAT_ERR_INVALID;
    if (!supported_d(d)) return RAT_ERR_UNSUPPORTED;
    if (pos0 < 0 || !std::isfinite(rope_base)) return RAT_ERR_INVALID;
    if (T == 0) return RAT_OK;
    if (!k || !v || !gate_logit || !k_rec || !v_rec) return RAT_ERR_INVALID;
    if (!aligned16(k) || !aligned16(v) || !aligned16(gate_logit) || !aligned16(k_rec) ||
        !aligned16(v_rec))
        return RAT_ERR_INVALID;
    if ((long long)B * H * T > (1ll << 40)) return RAT_ERR_UNSUPPORTED;
    const size_t need = recur_workspace_bytes(B * H, T, d, dtype);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return RAT_ERR_WORKSPACE;

    RecurParams p;
    std::memset(&p, 0, sizeof(p));
    p.k = k; p.v = v; p.a = gate_logit;
    p.h0k = h0_k; p.h0v = h0_v;
    p.yk = k_rec; p.yv = v_rec;
    p.hTk = hT_k; p.hTv = hT_v;
    p.BH = B * H; p.T = T; p.d = d;
    const int tc = recur_chunk_rows(d, dtype);
    p.nchunks = (T + tc - 1) / tc;
    p.pos0 = pos0;
    p.reset = reset_every;
    p.rope = rope_base > 0.f ? 1 : 0;
    p.fault_chunk = g_fault_chunk;
    p.wait_ns = g_fault_chunk >= 0 ? g_fault_wait_ns : kWaitLimitNs;
    g_fault_chunk = -1;
    uint8_t *w = static_cast<uint8_t *>(ws);
    const size_t nch = (size_t)p.BH * p.nchunks;
    p.hdr = reinterpret_cast<WsHeader *>(w);
    p.agg = reinterpret_cast<uint64_t *>(w + sizeof(WsHeader));
    p.pre = reinterpret_cast<uint64_t *>(w + sizeof(WsHeader) + align256(nch * 3 * d * 8));
    if (p.rope) {
        rope_theta(rope_base, d, p.theta);
        for (int c = 0; c < 64; ++c) {
            p.theta_f[c] = (float)p.theta[c];
            p.step_cos[c] = (float)std::cos(p.theta[c]);
            p.step_sin[c] = (float)std::sin(p.theta[c]);
        }
        p.rope_f32 = (dtype == RAT_BF16 && pos0 + (int64_t)T <= 8192) ? 1 : 0;
    }
    return launch_recur(p, dtype, stream);
}
}  // namespace

namespace {
int recur_backward(const void *k, const void *v, const void *gate_logit, const float *h0_k,
                   const float *h0_v, const void *k_rec, const void *v_rec, const void *dk_rec,
                   const void *dv_rec, const float *dhT_k, const float *dhT_v, void *dk, void *dv,
                   void *dgate_logit, float *dh0_k, float *dh0_v, int B, int H, int T, int d,
                   int dtype, int64_t pos0, int64_t L, float rope_base, void *ws, size_t ws_bytes,
                   void *stream) {
    if (B < 1 || H < 1 || T < 0 || !valid_dtype(dtype) || L < 0) return RAT_ERR_INVALID;
    if (!supported_d(d)) return RAT_ERR_UNSUPPORTED;
    if (pos0 < 0 || !std::isfinite(rope_base)) return RAT_ERR_INVALID;
    if (T == 0) return RAT_OK;
    const void *req[] = {k, v, gate_logit, k_rec, v_rec, dk_rec, dv_rec, dk, dv, dgate_logit};
    for (const void *q : req)
        if (!q || !aligned16(q)) return RAT_ERR_INVALID;
    if ((long long)B * H * T > (1ll << 40)) return RAT_ERR_UNSUPPORTED;
    const size_t need = recur_bwd_workspace_bytes(B * H, T, d);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return RAT_ERR_WORKSPACE;
    RecurBwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.k = k; p.v = v; p.a = gate_logit; p.yk = k_rec; p.yv = v_rec; p.dyk = dk_rec; p.dyv = dv_rec;
    p.h0k = h0_k; p.h0v = h0_v; p.dhTk = dhT_k; p.dhTv = dhT_v;
    p.dk = dk; p.dv = dv; p.da = dgate_logit; p.dh0k = dh0_k; p.dh0v = dh0_v;
    p.BH = B * H; p.T = T; p.d = d;
    const int tc = recur_bwd_chunk_rows(d, dtype);
    if ((long long)B * H * ((T + tc - 1) / tc) > 0x7fffffffll) return RAT_ERR_UNSUPPORTED;
    p.nch = (T + tc - 1) / tc;
    p.pos0 = pos0;
    p.reset = L;
    p.rope = rope_base > 0.f ? 1 : 0;
    uint8_t *w = static_cast<uint8_t *>(ws);
    p.hdr = reinterpret_cast<WsHeader *>(w);
    p.agg = reinterpret_cast<uint64_t *>(w + sizeof(WsHeader));
    p.pre = reinterpret_cast<uint64_t *>(w + sizeof(WsHeader) + align256((size_t)p.BH * p.nch * 3 * d * 8));
    p.fault_chunk = g_fault_chunk;
    p.wait_ns = g_fault_chunk >= 0 ? g_fault_wait_ns : kWaitLimitNs;
    g_fault_chunk = -1;
    if (p.rope) {
        rope_theta(rope_base, d, p.theta);
        for (int c = 0; c < 64; ++c) {
            p.theta_f[c] = (float)p.theta[c];
            p.step_cos[c] = (float)std::cos(p.theta[c]);
            p.step_sin[c] = (float)std::sin(p.theta[c]);
        }
        p.rope_f32 = (dtype == RAT_BF16 && pos0 + (int64_t)T <= 8192) ? 1 : 0;
    }
    return launch_recur_bwd(p, dtype, stream);
}
}  // namespace

extern "C" {

int rat_recur_prefill(const void *k, const void *v, const void *gate_logit, const float *h0_k,
                      const float *h0_v, void *k_rec, void *v_rec, float *hT_k, float *hT_v,
                      int B, int H, int T, int d, int dtype, int64_t pos0, float rope_base,
                      void *ws, size_t ws_bytes, void *stream) {
    return recur_prefill(k, v, gate_logit, h0_k, h0_v, k_rec, v_rec, hT_k, hT_v, B, H, T, d,
                         dtype, pos0, 0, rope_base, ws, ws_bytes, stream);
}

size_t rat_recur_backward_workspace_bytes(int B, int H, int T, int d) {
    if (B < 1 || H < 1 || T < 0 || !supported_d(d)) return 0;
    return recur_bwd_workspace_bytes(B * H, T, d);
}

int rat_recur_backward(const void *k, const void *v, const void *gate_logit, const float *h0_k,
                       const float *h0_v, const void *k_rec, const void *v_rec,
                       const void *dk_rec, const void *dv_rec, const float *dhT_k,
                       const float *dhT_v, void *dk, void *dv, void *dgate_logit, float *dh0_k,
                       float *dh0_v, int B, int H, int T, int d, int dtype, int64_t pos0,
                       float rope_base, void *ws, size_t ws_bytes, void *stream) {
    return recur_backward(k, v, gate_logit, h0_k, h0_v, k_rec, v_rec, dk_rec, dv_rec, dhT_k,
                          dhT_v, dk, dv, dgate_logit, dh0_k, dh0_v, B, H, T, d, dtype, pos0, 0,
                          rope_base, ws, ws_bytes, stream);
}

int rat_recur_backward_local(const void *k, const void *v, const void *gate_logit,
                             const float *h0_k, const float *h0_v, const void *k_rec,
                             const void *v_rec, const void *dk_rec, const void *dv_rec,
                             const float *dhT_k, const float *dhT_v, void *dk, void *dv,
                             void *dgate_logit, float *dh0_k, float *dh0_v, int B, int H, int T,
                             int d, int dtype, int64_t pos0, int64_t L, float rope_base, void *ws,
                             size_t ws_bytes, void *stream) {
    if (L < 1) return RAT_ERR_INVALID;
    return recur_backward(k, v, gate_logit, h0_k, h0_v, k_rec, v_rec, dk_rec, dv_rec, dhT_k,
                          dhT_v, dk, dv, dgate_logit, dh0_k, dh0_v, B, H, T, d, dtype, pos0, L,
                          rope_base, ws, ws_bytes, stream);
}

int rat_recur_prefill_window(const void *k, const void *v, const void *gate_logit,
                             const void *prev_k, const void *prev_v, const void *prev_gate_logit,
                             void *k_rec, void *v_rec, int B, int H, int T, int d, int dtype,
                             int64_t pos0, int64_t Lw, float rope_base, void *ws, size_t ws_bytes,
                             void *stream) {
    if (B < 1 || H < 1 || T < 0 || !valid_dtype(dtype) || Lw < 1) return RAT_ERR_INVALID;
    if (!supported_d(d) || Lw != kWindowRows) return RAT_ERR_UNSUPPORTED;
    if (pos0 < 0 || !std::isfinite(rope_base)) return RAT_ERR_INVALID;
    const int nprev = (prev_k != nullptr) + (prev_v != nullptr) + (prev_gate_logit != nullptr);
    if (nprev != 0 && nprev != 3) return RAT_ERR_INVALID;
    if (T == 0) return RAT_OK;
    if (!k || !v || !gate_logit || !k_rec || !v_rec) return RAT_ERR_INVALID;
    if (!aligned16(k) || !aligned16(v) || !aligned16(gate_logit) || !aligned16(k_rec) ||
        !aligned16(v_rec) || (nprev && (!aligned16(prev_k) || !aligned16(prev_v) ||
                                        !aligned16(prev_gate_logit))))
        return RAT_ERR_INVALID;
    if ((long long)B * H * T > (1ll << 40)) return RAT_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return RAT_ERR_WORKSPACE;
    WindowParams p;
    std::memset(&p, 0, sizeof(p));
    p.k = k; p.v = v; p.a = gate_logit;
    p.pk = prev_k; p.pv = prev_v; p.pa = prev_gate_logit;
    p.yk = k_rec; p.yv = v_rec;
    p.BH = B * H; p.T = T; p.d = d;
    p.nblk = (T + kWindowRows - 1) / kWindowRows;
    p.pos0 = pos0;
    p.rope = rope_base > 0.f ? 1 : 0;
    p.hdr = static_cast<WsHeader *>(ws);
    if (p.rope) {
        rope_theta(rope_base, d, p.theta);
        for (int c = 0; c < 64; ++c) {
            p.theta_f[c] = (float)p.theta[c];
            p.step_cos[c] = (float)std::cos(p.theta[c]);
            p.step_sin[c] = (float)std::sin(p.theta[c]);
        }
        p.rope_f32 = (dtype == RAT_BF16 && pos0 + (int64_t)T <= 8192) ? 1 : 0;
    }
    return launch_window(p, dtype, stream);
}

int rat_recur_backward_window(const void *k, const void *v, const void *gate_logit,
                              const void *prev_k, const void *prev_v,
                              const void *prev_gate_logit, const void *dk_rec,
                              const void *dv_rec, void *dk, void *dv, void *dgate_logit,
                              void *dprev_k, void *dprev_v, void *dprev_gate_logit, int B, int H,
                              int T, int d, int dtype, int64_t pos0, int64_t Lw, float rope_base,
                              void *stream) {
    if (B < 1 || H < 1 || T < 0 || !valid_dtype(dtype) || Lw < 1) return RAT_ERR_INVALID;
    if (!supported_d(d) || Lw != kWindowRows) return RAT_ERR_UNSUPPORTED;
    if (pos0 < 0 || !std::isfinite(rope_base)) return RAT_ERR_INVALID;
    const int nprev = (prev_k != nullptr) + (prev_v != nullptr) + (prev_gate_logit != nullptr);
    const int ndprev = (dprev_k != nullptr) + (dprev_v != nullptr) + (dprev_gate_logit != nullptr);
    if ((nprev != 0 && nprev != 3) || (ndprev != 0 && ndprev != 3) || (ndprev && !nprev))
        return RAT_ERR_INVALID;
    if (T == 0) return RAT_OK;
    if (!k || !v || !gate_logit || !dk_rec || !dv_rec || !dk || !dv || !dgate_logit)
        return RAT_ERR_INVALID;
    const void *ptrs[] = {k, v, gate_logit, dk_rec, dv_rec, dk, dv, dgate_logit, prev_k, prev_v,
                          prev_gate_logit, dprev_k, dprev_v, dprev_gate_logit};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return RAT_ERR_INVALID;
    if ((long long)B * H * T > (1ll << 40) || (long long)B * H * (d / 32) * (T / kWindowRows + 2) >= (1ll << 31))
        return RAT_ERR_UNSUPPORTED;
    WindowBwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.k = k; p.v = v; p.a = gate_logit;
    p.pk = prev_k; p.pv = prev_v; p.pa = prev_gate_logit;
    p.dyk = dk_rec; p.dyv = dv_rec;
    p.dk = dk; p.dv = dv; p.da = dgate_logit;
    p.dpk = dprev_k; p.dpv = dprev_v; p.dpa = dprev_gate_logit;
    p.BH = B * H; p.T = T; p.d = d;
    p.nblk = (T + kWindowRows - 1) / kWindowRows;
    p.pos0 = pos0;
    p.rope = rope_base > 0.f ? 1 : 0;
    if (p.rope) {
        rope_theta(rope_base, d, p.theta);
        for (int c = 0; c < 64; ++c) {
            p.theta_f[c] = (float)p.theta[c];
            p.step_cos[c] = (float)std::cos(p.theta[c]);
            p.step_sin[c] = (float)std::sin(p.theta[c]);
            p.step64_cos[c] = (float)std::cos(kWindowRows * p.theta[c]);
            p.step64_sin[c] = (float)std::sin(kWindowRows * p.theta[c]);
        }
        p.rope_f32 = (dtype == RAT_BF16 && pos0 + (int64_t)T <= 8192) ? 1 : 0;
    }
    return launch_window_bwd(p, dtype, stream);
}

int rat_recur_prefill_local(const void *k, const void *v, const void *gate_logit,
                            const float *h0_k, const float *h0_v, void *k_rec, void *v_rec,
                            float *hT_k, float *hT_v, int B, int H, int T, int d, int dtype,
                            int64_t pos0, int64_t L, float rope_base, void *ws, size_t ws_bytes,
                            void *stream) {
    if (L < 1) return RAT_ERR_INVALID;
    return recur_prefill(k, v, gate_logit, h0_k, h0_v, k_rec, v_rec, hT_k, hT_v, B, H, T, d,
                         dtype, pos0, L, rope_base, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------------------ attention
}  // extern "C"

namespace {
int attn_prefill(const void *q, const void *k_rec, const void *v_rec, void *o, int B, int H,
                 int T, int d, int dtype, int D, int W, const int32_t *D_per_head, int n_sink,
                 int top_k, float *lse, int64_t pos0, float rope_base, float scale,
                 void *stream) {
    if (B < 1 || H < 1 || T < 0 || !valid_dtype(dtype) || W < 0 || pos0 < 0 || n_sink < 0 ||
        top_k < 0)
        return RAT_ERR_INVALID;
    if (top_k > 16) return RAT_ERR_UNSUPPORTED;
    if (!supported_d(d) || H > kMaxHeads) return RAT_ERR_UNSUPPORTED;
    if (!std::isfinite(rope_base) || !std::isfinite(scale)) return RAT_ERR_INVALID;
    if (!D_per_head && D < 1) return RAT_ERR_INVALID;
    if (D_per_head)
        for (int h = 0; h < H; ++h)
            if (D_per_head[h] < 1) return RAT_ERR_INVALID;
    if (T == 0) return RAT_OK;
    if (!q || !k_rec || !v_rec || !o) return RAT_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k_rec) || !aligned16(v_rec) || !aligned16(o)) return RAT_ERR_INVALID;
    if ((long long)B * H > 65535 || T > (1 << 30)) return RAT_ERR_UNSUPPORTED;
    const float sc = scale > 0.f ? scale : (float)(1.0 / std::sqrt((double)d));
    const float scale_log2 = sc * 1.4426950408889634f;

    int32_t Dh[kMaxHeads];
    for (int h = 0; h < H; ++h) Dh[h] = D_per_head ? D_per_head[h] : D;

    // the tensor-core kernel takes sinks as one extra key block when no chunk end is a sink
    bool sinks_fit = n_sink <= 64;
    for (int h = 0; h < H; ++h)
        if (Dh[h] > 1 && Dh[h] <= n_sink) sinks_fit = false;
    // top-k chunk selection runs there too when there are no sinks and the sequence's 64-key
    // blocks fit the kernel's block bitmap
    const bool topk_fits = top_k == 0 || (n_sink == 0 && T <= 65536);
    if (dtype == RAT_BF16 && d == 128 && topk_fits && (n_sink == 0 || sinks_fit)) {
        AttnSm100Args a;
        std::memset(&a, 0, sizeof(a));
        a.q = q; a.k = k_rec; a.v = v_rec; a.o = o;
        a.B = B; a.H = H; a.T = T; a.d = d; a.W = W;
        a.pos0 = pos0;
        a.rope = rope_base > 0.f ? 1 : 0;
        a.scale_log2 = scale_log2;
        a.Dh = Dh;
        a.n_sink = n_sink;
        a.top_k = top_k;
        a.lse = lse;
        if (a.rope) rope_theta(rope_base, d, a.theta);
        return launch_attn_sm100(a, stream);
    }
    AttnSimtParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q; p.k = k_rec; p.v = v_rec; p.o = o;
    p.B = B; p.H = H; p.T = T; p.d = d; p.W = W;
    p.pos0 = pos0;
    p.rope = rope_base > 0.f ? 1 : 0;
    p.scale_log2 = scale_log2;
    p.n_sink = n_sink;
    p.top_k = top_k;
    p.lse = lse;
    for (int h = 0; h < H; ++h) p.Dh[h] = Dh[h];
    if (p.rope) rope_theta(rope_base, d, p.theta);
    return launch_attn_simt(p, dtype, stream);
}
}  // namespace

extern "C" {

int rat_dilated_attn_prefill(const void *q, const void *k_rec, const void *v_rec, void *o, int B,
                             int H, int T, int d, int dtype, int D, int W,
                             const int32_t *D_per_head, int64_t pos0, float rope_base,
                             float scale, void *stream) {
    return attn_prefill(q, k_rec, v_rec, o, B, H, T, d, dtype, D, W, D_per_head, 0, 0, nullptr,
                        pos0, rope_base, scale, stream);
}

int rat_dilated_attn_prefill_sinks(const void *q, const void *k_rec, const void *v_rec, void *o,
                                   int B, int H, int T, int d, int dtype, int D, int W,
                                   const int32_t *D_per_head, int n_sink, int64_t pos0,
                                   float rope_base, float scale, void *stream) {
    return attn_prefill(q, k_rec, v_rec, o, B, H, T, d, dtype, D, W, D_per_head, n_sink, 0,
                        nullptr, pos0, rope_base, scale, stream);
}

int rat_dilated_attn_prefill_topk(const void *q, const void *k_rec, const void *v_rec, void *o,
                                  int B, int H, int T, int d, int dtype, int D, int W,
                                  const int32_t *D_per_head, int n_sink, int top_k, int64_t pos0,
                                  float rope_base, float scale, void *stream) {
    return attn_prefill(q, k_rec, v_rec, o, B, H, T, d, dtype, D, W, D_per_head, n_sink, top_k,
                        nullptr, pos0, rope_base, scale, stream);
}

int rat_dilated_attn_prefill_ex(const void *q, const void *k_rec, const void *v_rec, void *o,
                                int B, int H, int T, int d, int dtype, int D, int W,
                                const int32_t *D_per_head, int64_t pos0, float rope_base,
                                float scale, const rat_attn_options *opt, void *stream) {
    if (!opt)
        return attn_prefill(q, k_rec, v_rec, o, B, H, T, d, dtype, D, W, D_per_head, 0, 0, nullptr,
                            pos0, rope_base, scale, stream);
    if (opt->lse && (reinterpret_cast<uintptr_t>(opt->lse) & 3u)) return RAT_ERR_INVALID;
    return attn_prefill(q, k_rec, v_rec, o, B, H, T, d, dtype, D, W, D_per_head, opt->n_sink,
                        opt->top_k, opt->lse, pos0, rope_base, scale, stream);
}

size_t rat_dilated_attn_backward_workspace_bytes(int B, int H, int T, int d, int dtype) {
    if (B < 1 || H < 1 || T < 0 || !supported_d(d) || !valid_dtype(dtype)) return 0;
    return attn_bwd_workspace_bytes(B, H, T, d, dtype);
}

int rat_dilated_attn_backward(const void *q, const void *k_rec, const void *v_rec, const void *o,
                              const void *dO, void *dq, void *dk_rec, void *dv_rec, int B, int H,
                              int T, int d, int dtype, int D, int W, const int32_t *D_per_head,
                              int n_sink, const float *lse, int64_t pos0, float rope_base,
                              float scale, void *ws, size_t ws_bytes, void *stream) {
    if (B < 1 || H < 1 || T < 0 || !valid_dtype(dtype) || W < 0 || pos0 < 0 || n_sink < 0)
        return RAT_ERR_INVALID;
    if (!supported_d(d) || H > kMaxHeads) return RAT_ERR_UNSUPPORTED;
    if (!std::isfinite(rope_base) || !std::isfinite(scale)) return RAT_ERR_INVALID;
    if (!D_per_head && D < 1) return RAT_ERR_INVALID;
    if (D_per_head)
        for (int h = 0; h < H; ++h)
            if (D_per_head[h] < 1) return RAT_ERR_INVALID;
    if (T == 0) return RAT_OK;
    const void *req[] = {q, k_rec, v_rec, o, dO, dq, dk_rec, dv_rec};
    for (const void *x : req)
        if (!x || !aligned16(x)) return RAT_ERR_INVALID;
    if ((long long)B * H > 65535 || T > (1 << 30)) return RAT_ERR_UNSUPPORTED;
    const size_t need = attn_bwd_workspace_bytes(B, H, T, d, dtype);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return RAT_ERR_WORKSPACE;
    AttnBwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q; p.k = k_rec; p.v = v_rec; p.o = o; p.dO = dO;
    p.dq = dq; p.dk = dk_rec; p.dv = dv_rec;
    const size_t rows = (size_t)B * H * T;
    p.hdr = static_cast<WsHeader *>(ws);
    uint8_t *w = static_cast<uint8_t *>(ws) + sizeof(WsHeader);
    p.qh = w;
    w += align256(rows * d * (dtype == RAT_F32 ? 4 : 2));
    p.lse = lse ? const_cast<float *>(lse) : reinterpret_cast<float *>(w);
    p.lse_given = lse ? 1 : 0;
    w += align256(rows * 4);
    p.delta = reinterpret_cast<float *>(w);
    p.B = B; p.H = H; p.T = T; p.d = d; p.W = W; p.n_sink = n_sink;
    p.pos0 = pos0;
    p.rope = rope_base > 0.f ? 1 : 0;
    p.scale = scale > 0.f ? scale : (float)(1.0 / std::sqrt((double)d));
    p.scale_log2 = p.scale * 1.4426950408889634f;
    for (int h = 0; h < H; ++h) p.Dh[h] = D_per_head ? D_per_head[h] : D;
    if (p.rope) rope_theta(rope_base, d, p.theta);
    return launch_attn_bwd(p, dtype, stream);
}

int rat_attn_sync_status(void *stream) { return attn_error_word(stream, true); }

uint32_t rat_attn_error_site(void) { return attn_error_where(); }

uint32_t rat_attn_error_waiting(void) { return attn_error_waiting(); }


int rat_set_attn_block_keys(int block_keys) {
    if (block_keys != 0 && block_keys != 64 && block_keys != 128) return RAT_ERR_INVALID;
    g_attn_block_keys = block_keys;
    return RAT_OK;
}

// ------------------------------------------------------------------------------ cache
int rat_kv_cache_bytes(const rat_kv_cache *c, size_t *dil_bytes, size_t *win_bytes,
                       size_t *state_bytes) {
    if (!valid_cache(c)) return RAT_ERR_INVALID;
    const size_t row = (size_t)c->d * esize(c->dtype);
    const long long total = total_capacity(c->H, c->Tcap, c->D, nullptr);
    if (dil_bytes) *dil_bytes = (size_t)c->B * total * row;
    if (win_bytes) *win_bytes = (size_t)c->B * c->H * c->W * row;
    if (state_bytes) *state_bytes = (size_t)c->B * c->H * c->d * sizeof(float);
    return RAT_OK;
}

size_t rat_kv_raw_bytes(const rat_kv_cache *c) {
    if (!valid_cache(c) || c->window_rec == 0) return 0;
    return (size_t)c->B * c->H * c->window_rec * c->d * esize(c->dtype);
}

namespace {
// the chunk ends, ring and sink rows of T positions (and the state when hT is given)
int compress_common(const void *k_rec, const void *v_rec, const float *hT_k, const float *hT_v,
                    int T, rat_kv_cache *c, void *stream) {
    if (!valid_cache(c) || T < 0) return RAT_ERR_INVALID;
    if (c->pos < 0 || c->pos + T > c->Tcap) return RAT_ERR_INVALID;
    if (T == 0) return RAT_OK;
    if (!k_rec || !v_rec || !c->k_dil || !c->v_dil || !c->h_k || !c->h_v) return RAT_ERR_INVALID;
    if (c->W > 0 && (!c->k_win || !c->v_win)) return RAT_ERR_INVALID;
    if (c->n_sink > 0 && (!c->k_sink || !c->v_sink || !aligned16(c->k_sink) || !aligned16(c->v_sink)))
        return RAT_ERR_INVALID;
    if (!aligned16(k_rec) || !aligned16(v_rec) || !aligned16(c->k_dil) || !aligned16(c->v_dil) ||
        (c->W > 0 && (!aligned16(c->k_win) || !aligned16(c->v_win))))
        return RAT_ERR_INVALID;
    CompressParams p;
    std::memset(&p, 0, sizeof(p));
    p.k = k_rec; p.v = v_rec; p.hTk = hT_k; p.hTv = hT_v;
    p.kdil = c->k_dil; p.vdil = c->v_dil; p.kwin = c->k_win; p.vwin = c->v_win;
    p.hk = c->h_k; p.hv = c->h_v;
    p.B = c->B; p.H = c->H; p.T = T; p.d = c->d; p.W = c->W; p.Tcap = c->Tcap;
    p.esize = esize(c->dtype);
    p.pos0 = c->pos;
    p.ksink = c->k_sink; p.vsink = c->v_sink; p.n_sink = c->n_sink;
    for (int h = 0; h < c->H; ++h) p.Dh[h] = c->D[h];
    p.total_cap = total_capacity(c->H, c->Tcap, c->D, p.off);
    return launch_compress(p, stream);
}
}  // namespace

int rat_kv_compress(const void *k_rec, const void *v_rec, const float *hT_k, const float *hT_v,
                    int T, rat_kv_cache *c, void *stream) {
    if (!valid_cache(c) || c->window_rec != 0) return RAT_ERR_INVALID;
    const int st = compress_common(k_rec, v_rec, hT_k, hT_v, T, c, stream);
    if (st == RAT_OK) c->pos += T;
    return st;
}

int rat_kv_compress_window(const void *k_rec, const void *v_rec, const void *k, const void *v,
                           const void *gate_logit, int T, rat_kv_cache *c, void *stream) {
    if (!valid_cache(c) || c->window_rec == 0 || T < 0 || !raw_rings_ok(c)) return RAT_ERR_INVALID;
    if (c->pos < 0 || c->pos + T > c->Tcap) return RAT_ERR_INVALID;
    if (T == 0) return RAT_OK;
    if (!k || !v || !gate_logit || !aligned16(k) || !aligned16(v) || !aligned16(gate_logit))
        return RAT_ERR_INVALID;
    int st = compress_common(k_rec, v_rec, nullptr, nullptr, T, c, stream);
    if (st != RAT_OK) return st;
    // raw rows of the last min(T, Lw) positions P .. pos+T-1 into slots p mod Lw: at most two
    // runs of slots (before and after the wrap), each one strided copy over every (b, h) slice
    const long long Lw = c->window_rec, end = c->pos + T, first = end - (T < Lw ? T : Lw);
    const size_t row = (size_t)c->d * esize(c->dtype);
    const void *src[3] = {k, v, gate_logit};
    void *dst[3] = {c->k_raw, c->v_raw, c->a_raw};
    const size_t slices = (size_t)c->B * c->H;
    for (long long p0 = first; p0 < end;) {
        const long long slot = p0 % Lw;
        const long long n = std::min(end - p0, Lw - slot);        // up to the end of the ring
        for (int i = 0; i < 3; ++i) {
            const uint8_t *s = static_cast<const uint8_t *>(src[i]) + (size_t)(p0 - c->pos) * row;
            uint8_t *d = static_cast<uint8_t *>(dst[i]) + (size_t)slot * row;
            if (cudaMemcpy2DAsync(d, (size_t)Lw * row, s, (size_t)T * row, (size_t)n * row, slices,
                                  cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)) != cudaSuccess)
                return RAT_ERR_CUDA;
        }
        p0 += n;
    }
    c->pos += T;
    return RAT_OK;
}

// ------------------------------------------------------------------------------ decode
size_t rat_decode_workspace_bytes(const rat_kv_cache *c) {
    if (!valid_cache(c)) return 0;
    const int s = decode_splits(c->B, c->H, c->Tcap, c->D, c->W);
    return decode_workspace_bytes(c->B, c->H, c->d, s);
}

// ------------------------------------------------------------------------------ paged cache
int rat_paged_kv_compress(const void *k_rec, const void *v_rec, const float *hT_k,
                          const float *hT_v, int T, int b, int64_t pos0,
                          rat_paged_kv_cache *c, void *ws, size_t ws_bytes, void *stream) {
    if (!valid_paged_cache(c) || T < 0 || b < 0 || b >= c->B || pos0 < 0) return RAT_ERR_INVALID;
    if (!ws || ws_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return RAT_ERR_WORKSPACE;
    if (T == 0) return RAT_OK;
    if (!k_rec || !v_rec || !aligned16(k_rec) || !aligned16(v_rec)) return RAT_ERR_INVALID;
    CompressParams p;
    std::memset(&p, 0, sizeof(p));
    p.k = k_rec; p.v = v_rec; p.hTk = hT_k; p.hTv = hT_v;
    p.kdil = c->k_pool; p.vdil = c->v_pool; p.kwin = c->k_win; p.vwin = c->v_win;
    p.hk = c->h_k; p.hv = c->h_v;
    p.B = 1; p.H = c->H; p.T = T; p.d = c->d; p.W = c->W;
    p.esize = esize(c->dtype);
    p.pos0 = pos0;
    for (int h = 0; h < c->H; ++h) p.Dh[h] = c->D[h];
    p.page_table = c->page_table;
    p.page_shift = log2_exact(c->page_entries);
    p.max_pages = c->max_pages;
    p.n_pages = c->n_pages;
    p.seq = b;
    p.seq_pos = reinterpret_cast<long long *>(c->pos);
    p.hdr = static_cast<WsHeader *>(ws);
    return launch_compress(p, stream);
}

size_t rat_paged_decode_workspace_bytes(const rat_paged_kv_cache *c) {
    if (!valid_paged_cache(c)) return 0;
    const long long keys = (long long)c->max_pages * c->page_entries + c->W;
    return decode_workspace_bytes(c->B, c->H, c->d, decode_splits_for_keys(c->B, c->H, keys));
}

int rat_dilated_decode_paged(const void *q, const void *k, const void *v, const void *gate_logit,
                             rat_paged_kv_cache *c, void *o, float rope_base, float scale,
                             void *ws, size_t ws_bytes, void *stream) {
    if (!valid_paged_cache(c)) return RAT_ERR_INVALID;
    if (c->dtype != RAT_BF16) return RAT_ERR_UNSUPPORTED;
    if (!q || !k || !v || !gate_logit || !o) return RAT_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate_logit) || !aligned16(o))
        return RAT_ERR_INVALID;
    if (!std::isfinite(rope_base) || !std::isfinite(scale)) return RAT_ERR_INVALID;
    if ((long long)c->B * c->H > 65535) return RAT_ERR_UNSUPPORTED;
    const long long keys = (long long)c->max_pages * c->page_entries + c->W;
    const int splits = decode_splits_for_keys(c->B, c->H, keys);
    const size_t need = decode_workspace_bytes(c->B, c->H, c->d, splits);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return RAT_ERR_WORKSPACE;

    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q; p.k = k; p.v = v; p.a = gate_logit; p.o = o;
    p.kdil = c->k_pool; p.vdil = c->v_pool; p.kwin = c->k_win; p.vwin = c->v_win;
    p.hk = c->h_k; p.hv = c->h_v;
    p.B = c->B; p.H = c->H; p.d = c->d; p.W = c->W; p.splits = splits;
    p.reset = c->reset_every;
    for (int h = 0; h < c->H; ++h) p.Dh[h] = c->D[h];
    p.rope = rope_base > 0.f ? 1 : 0;
    const float sc = scale > 0.f ? scale : (float)(1.0 / std::sqrt((double)c->d));
    p.scale_log2 = sc * 1.4426950408889634f;
    uint8_t *w = static_cast<uint8_t *>(ws);
    const size_t bh = (size_t)c->B * c->H;
    p.hdr = reinterpret_cast<WsHeader *>(w);
    size_t off = sizeof(WsHeader);
    p.tickets = reinterpret_cast<uint32_t *>(w + off);
    off += align256(bh * 4);
    p.part_ml = reinterpret_cast<float *>(w + off);
    off += align256(bh * splits * 2 * 4);
    p.part_o = reinterpret_cast<float *>(w + off);
    off += align256(bh * splits * c->d * 4);
    p.seq_ticket = reinterpret_cast<uint32_t *>(w + off);
    p.seq_pos = reinterpret_cast<long long *>(c->pos);
    p.page_table = c->page_table;
    p.page_shift = log2_exact(c->page_entries);
    p.max_pages = c->max_pages;
    p.n_pages = c->n_pages;
    if (p.rope) rope_theta(rope_base, c->d, p.theta);
    return launch_decode(p, c->dtype, stream, true);
}

int rat_dilated_decode(const void *q, const void *k, const void *v, const void *gate_logit,
                       rat_kv_cache *c, void *o, float rope_base, float scale, void *ws,
                       size_t ws_bytes, void *stream) {
    if (!valid_cache(c) || !raw_rings_ok(c)) return RAT_ERR_INVALID;
    if (c->dtype != RAT_BF16) return RAT_ERR_UNSUPPORTED;
    if (!q || !k || !v || !gate_logit || !o) return RAT_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate_logit) || !aligned16(o))
        return RAT_ERR_INVALID;
    if (!c->k_dil || !c->v_dil || !c->h_k || !c->h_v) return RAT_ERR_INVALID;
    if (c->W > 0 && (!c->k_win || !c->v_win)) return RAT_ERR_INVALID;
    if (c->n_sink > 0 && (!c->k_sink || !c->v_sink || !aligned16(c->k_sink) || !aligned16(c->v_sink)))
        return RAT_ERR_INVALID;
    if (c->pos < 0 || c->pos >= c->Tcap) return RAT_ERR_INVALID;
    if (!std::isfinite(rope_base) || !std::isfinite(scale)) return RAT_ERR_INVALID;
    if ((long long)c->B * c->H > 65535) return RAT_ERR_UNSUPPORTED;
    const int splits = decode_splits(c->B, c->H, c->Tcap, c->D, c->W);
    const size_t need = decode_workspace_bytes(c->B, c->H, c->d, splits);
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return RAT_ERR_WORKSPACE;

    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = q; p.k = k; p.v = v; p.a = gate_logit; p.o = o;
    p.kdil = c->k_dil; p.vdil = c->v_dil; p.kwin = c->k_win; p.vwin = c->v_win;
    p.hk = c->h_k; p.hv = c->h_v;
    p.B = c->B; p.H = c->H; p.d = c->d; p.W = c->W; p.Tcap = c->Tcap; p.splits = splits;
    p.t = c->pos;
    p.reset = c->reset_every;
    p.ksink = c->k_sink; p.vsink = c->v_sink; p.n_sink = c->n_sink;
    p.window_rec = c->window_rec;
    p.kraw = c->k_raw; p.vraw = c->v_raw; p.araw = c->a_raw;
    for (int h = 0; h < c->H; ++h) p.Dh[h] = c->D[h];
    p.total_cap = total_capacity(c->H, c->Tcap, c->D, p.off);
    p.rope = rope_base > 0.f ? 1 : 0;
    const float sc = scale > 0.f ? scale : (float)(1.0 / std::sqrt((double)c->d));
    p.scale_log2 = sc * 1.4426950408889634f;
    uint8_t *w = static_cast<uint8_t *>(ws);
    const size_t bh = (size_t)c->B * c->H;
    p.hdr = reinterpret_cast<WsHeader *>(w);
    p.tickets = reinterpret_cast<uint32_t *>(w + sizeof(WsHeader));
    p.part_ml = reinterpret_cast<float *>(w + sizeof(WsHeader) + align256(bh * 4));
    p.part_o = reinterpret_cast<float *>(w + sizeof(WsHeader) + align256(bh * 4) + align256(bh * splits * 2 * 4));
    if (p.rope) rope_theta(rope_base, c->d, p.theta);
    const int st = launch_decode(p, c->dtype, stream);
    if (st == RAT_OK) c->pos += 1;
    return st;
}

}  // extern "C"
