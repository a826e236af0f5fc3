// attn_bwd.cu -- backward of the causal dilated attention (CUDA cores, float32 accumulation).
//
// The forward (RAT+ abstract; "RAT+ Deep Dive" sections 3.1 and 6): query t of head h attends
//   S(t) = { t-We < j <= t }  U  { j <= t-We : j mod D_h = D_h - 1 },   We = max(W, 1),
// plus, with n_sink > 0, the first n_sink positions (attention sinks, each key once),
// o_t = sum_{j in S(t)} p_tj v_j,  p_t = softmax_j(scale <q^_t, k~_j>),  q^ = RoPE(q).
// Its reverse-mode derivative, for upstream gradients dO:
//   dp_tj = <dO_t, v_j>,   ds_tj = p_tj (dp_tj - <dO_t, o_t>),
//   dq^_t = scale sum_j ds_tj k~_j,   dk~_j = scale sum_t ds_tj q^_t,   dv_j = sum_t p_tj dO_t,
//   dq = RoPE^T(dq^).
// Three launches, one warp per row, each lane holding d/32 consecutive channels:
//   prep : q^ = RoPE(q) (rounded to the dtype, as the attention's operand) and <dO_t, o_t>;
//   dq   : per query, the key set walked twice -- once for the softmax denominator (kept for
//          the next launch), once for dq;
//   dkv  : per key, the queries whose key set holds it walked once: the window t in
//          [j, j + We - 1], and, for a chunk end (j mod D = D - 1), every t >= j + We; the
//          chunk ends are handed out first, so the long walks share CTAs.
// Each (query, key) pair is recomputed in both gradient launches; p comes from the stored
// denominator, so the two launches agree.  This is the plain CUDA-core path of the backward:
// dot products are warp reductions, four rows' loads in flight per warp.
#include <cstring>

#include "common.cuh"

namespace rat {

namespace {

// rotate-half RoPE of a lane's CPL channels (partner channel c +- d/2 lives 16 lanes away);
// sign = +1 for the rotation, -1 for its transpose
template <int DH>
RAT_DEVICE void rope_lane(const AttnBwdParams &p, long long pos, int lane, float sign, float *x) {
    constexpr int CPL = DH / 32;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        const int c = lane * CPL + j;
        float cs, sn;
        rope_cs(pos, p.theta[c % (DH / 2)], cs, sn);
        sn *= sign;
        const float partner = __shfl_xor_sync(0xffffffffu, x[j], 16);
        x[j] = c < DH / 2 ? x[j] * cs - partner * sn : x[j] * cs + partner * sn;
    }
}

constexpr int kRows = 4;        // rows (keys or queries) whose loads are issued together

}  // namespace

// q^ = RoPE(q) and Delta_t = dO_t . o_t.  One warp walks kPrepRows consecutive rows; lane l holds
// channels l*CPL .. l*CPL+CPL-1 (the rotate-half partner of channel c < d/2 sits in lane l ^ 16).
// The lane's angles are formed once at the warp's first row and advanced one position per row
// by a complex multiply with (cos theta, sin theta).
constexpr int kPrepRows = 16;

template <typename E, int DH>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __grid_constant__ AttnBwdParams p) {
    constexpr int CPL = DH / 32, EB = sizeof(E), ROWB = DH * EB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int t0 = (blockIdx.x * 8 + warp) * kPrepRows;
    if (t0 >= p.T) return;
    const int nr = min(kPrepRows, p.T - t0);
    const size_t off = ((size_t)bh * p.T + t0) * ROWB + lane * CPL * EB;
    const uint8_t *gq = static_cast<const uint8_t *>(p.q) + off;
    const uint8_t *go = static_cast<const uint8_t *>(p.o) + off;
    const uint8_t *gg = static_cast<const uint8_t *>(p.dO) + off;
    uint8_t *gh = static_cast<uint8_t *>(p.qh) + off;
    float cs[CPL], sn[CPL], sc[CPL], ss[CPL];
    if (p.rope) {
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            const double th = p.theta[(lane * CPL + j) % (DH / 2)];
            rope_cs(p.pos0 + t0, th, cs[j], sn[j]);
            rope_cs(1, th, sc[j], ss[j]);
        }
    }
    const bool first_half = lane < 16;
#pragma unroll 4
    for (int r = 0; r < nr; ++r) {
        float q[CPL], o[CPL], g[CPL];
        RowIO<E, CPL>::load(gq + (size_t)r * ROWB, q);
        RowIO<E, CPL>::load(go + (size_t)r * ROWB, o);
        RowIO<E, CPL>::load(gg + (size_t)r * ROWB, g);
        if (p.rope) {
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                const float partner = __shfl_xor_sync(0xffffffffu, q[j], 16);
                q[j] = first_half ? q[j] * cs[j] - partner * sn[j] : q[j] * cs[j] + partner * sn[j];
                const float nc = cs[j] * sc[j] - sn[j] * ss[j];     // one position on
                sn[j] = sn[j] * sc[j] + cs[j] * ss[j];
                cs[j] = nc;
            }
        }
        RowIO<E, CPL>::store(gh + (size_t)r * ROWB, q);
        float dot = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) dot = fmaf(g[j], o[j], dot);
        dot = warp_sum(dot);
        if (lane == 0) p.delta[(size_t)bh * p.T + t0 + r] = dot;
    }
}

template <typename E, int DH>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const __grid_constant__ AttnBwdParams p) {
    constexpr int CPL = DH / 32, EB = sizeof(E);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, h = bh % p.H;
    const int t = blockIdx.x * 8 + warp;
    if (t >= p.T) return;
    const int D = p.Dh[h];
    const int We = p.W > 1 ? p.W : 1;
    const size_t row = (size_t)bh * p.T;
    const uint8_t *kb = static_cast<const uint8_t *>(p.k) + row * DH * EB + lane * CPL * EB;
    const uint8_t *vb = static_cast<const uint8_t *>(p.v) + row * DH * EB + lane * CPL * EB;
    const size_t off = (row + t) * DH * EB + lane * CPL * EB;
    float q[CPL], g[CPL];
    RowIO<E, CPL>::load(static_cast<const uint8_t *>(p.qh) + off, q);
    RowIO<E, CPL>::load(static_cast<const uint8_t *>(p.dO) + off, g);
    const float delta = p.delta[row + t];

    const int w_lo = max(0, t - We + 1);
    const int n_win = t - w_lo + 1;
    const int n_dil = t - We + 1 >= D ? (t - We + 1) / D : 0;
    const int s_lim = min(p.n_sink, max(0, t - We + 1));     // sinks that are not chunk ends
    const int n_snk = D > 1 ? s_lim - s_lim / D : 0;
    const int n = n_win + n_dil + n_snk;
    auto key = [&](int idx) {
        if (idx < n_win) return w_lo + idx;
        if (idx < n_win + n_dil) return (idx - n_win) * D + D - 1;
        const int s = idx - n_win - n_dil;
        return s + s / (D - 1);
    };

    // pass 1: the softmax denominator (log2 units), unless the forward's is given
    float m = -INFINITY, l = 0.f;
    for (int base = 0; base < (p.lse_given ? 0 : n); base += kRows) {
        float kx[kRows][CPL];
#pragma unroll
        for (int u = 0; u < kRows; ++u)
            if (base + u < n) RowIO<E, CPL>::load(kb + (size_t)key(base + u) * DH * EB, kx[u]);
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            if (base + u < n) {
                float dot = 0.f;
#pragma unroll
                for (int j = 0; j < CPL; ++j) dot = fmaf(q[j], kx[u][j], dot);
                const float s = warp_sum(dot) * p.scale_log2;
                const float mn = fmaxf(m, s);
                l = fmaf(l, exp2f(m - mn), exp2f(s - mn));
                m = mn;
            }
        }
    }
    const float lse = p.lse_given ? p.lse[row + t] : m + log2f(l);
    // pass 2: dq^ = scale sum_j p_j (<dO, v_j> - delta) k_j
    float dq[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) dq[j] = 0.f;
    for (int base = 0; base < n; base += kRows) {
        float kx[kRows][CPL], vx[kRows][CPL];
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            if (base + u < n) {
                const size_t jr = (size_t)key(base + u) * DH * EB;
                RowIO<E, CPL>::load(kb + jr, kx[u]);
                RowIO<E, CPL>::load(vb + jr, vx[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            if (base + u < n) {
                float sd = 0.f, pd = 0.f;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    sd = fmaf(q[j], kx[u][j], sd);
                    pd = fmaf(g[j], vx[u][j], pd);
                }
                sd = warp_sum(sd);
                pd = warp_sum(pd);
                const float pj = exp2f(sd * p.scale_log2 - lse);
                const float ds = pj * (pd - delta);
#pragma unroll
                for (int j = 0; j < CPL; ++j) dq[j] = fmaf(ds, kx[u][j], dq[j]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < CPL; ++j) dq[j] *= p.scale;
    if (p.rope) rope_lane<DH>(p, p.pos0 + t, lane, -1.f, dq);
    RowIO<E, CPL>::store(static_cast<uint8_t *>(p.dq) + off, dq);
    if (lane == 0 && !p.lse_given) p.lse[row + t] = lse;
}

template <typename E, int DH>
__global__ void __launch_bounds__(256) attn_bwd_dkv_kernel(const __grid_constant__ AttnBwdParams p) {
    constexpr int CPL = DH / 32, EB = sizeof(E);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, h = bh % p.H;
    // warps take the chunk ends first (every query older than their window holds them; the
    // oldest, with the most queries, in the first CTAs), then the other keys (their window
    // only), so that a CTA's warps have like amounts of work
    const int kk = blockIdx.x * 8 + warp;
    if (kk >= p.T) return;
    const int D = p.Dh[h];
    const int n_ce = p.T / D;                              // chunk ends in the sequence
    int j;
    if (kk < n_ce) {
        j = kk * D + D - 1;
    } else {
        const int m = kk - n_ce;                           // the m-th key that is not a chunk end
        j = m + m / (D - 1);                               // (D > 1 here: with D = 1 all are)
    }
    const int We = p.W > 1 ? p.W : 1;
    const size_t row = (size_t)bh * p.T;
    const size_t off = (row + j) * DH * EB + lane * CPL * EB;
    float kx[CPL], vx[CPL];
    RowIO<E, CPL>::load(static_cast<const uint8_t *>(p.k) + off, kx);
    RowIO<E, CPL>::load(static_cast<const uint8_t *>(p.v) + off, vx);
    const uint8_t *qb = static_cast<const uint8_t *>(p.qh) + row * DH * EB + lane * CPL * EB;
    const uint8_t *gb = static_cast<const uint8_t *>(p.dO) + row * DH * EB + lane * CPL * EB;

    // queries holding key j: t in [j, j + We - 1] (window), then t >= j + We (chunk end or sink)
    const int n_win = min(We, p.T - j);
    const int n_dil = (j % D == D - 1 || j < p.n_sink) ? max(0, p.T - (j + We)) : 0;
    const int n = n_win + n_dil;
    float dk[CPL], dv[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) { dk[c] = 0.f; dv[c] = 0.f; }
    for (int base = 0; base < n; base += kRows) {
        float qx[kRows][CPL], gx[kRows][CPL], lse[kRows], dl[kRows];
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            if (base + u < n) {
                const int t = j + base + u;             // both parts are contiguous from j
                RowIO<E, CPL>::load(qb + (size_t)t * DH * EB, qx[u]);
                RowIO<E, CPL>::load(gb + (size_t)t * DH * EB, gx[u]);
                lse[u] = p.lse[row + t];
                dl[u] = p.delta[row + t];
            }
        }
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            if (base + u < n) {
                float sd = 0.f, pd = 0.f;
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    sd = fmaf(qx[u][c], kx[c], sd);
                    pd = fmaf(gx[u][c], vx[c], pd);
                }
                sd = warp_sum(sd);
                pd = warp_sum(pd);
                const float pj = exp2f(sd * p.scale_log2 - lse[u]);
                const float ds = pj * (pd - dl[u]);
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    dk[c] = fmaf(ds, qx[u][c], dk[c]);
                    dv[c] = fmaf(pj, gx[u][c], dv[c]);
                }
            }
        }
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) dk[c] *= p.scale;
    RowIO<E, CPL>::store(static_cast<uint8_t *>(p.dk) + off, dk);
    RowIO<E, CPL>::store(static_cast<uint8_t *>(p.dv) + off, dv);
}

size_t attn_bwd_workspace_bytes(int B, int H, int T, int d, int dtype) {
    const size_t rows = (size_t)B * H * T;
    return sizeof(WsHeader) + align256(rows * d * (dtype == RAT_F32 ? 4 : 2)) + 2 * align256(rows * 4);
}

template <typename E, int DH>
static int launch_bwd(const AttnBwdParams &p, cudaStream_t s) {
    dim3 grid((unsigned)((p.T + 7) / 8), (unsigned)(p.B * p.H));
    const dim3 pgrid((unsigned)((p.T + 8 * kPrepRows - 1) / (8 * kPrepRows)), (unsigned)(p.B * p.H));
    attn_bwd_prep_kernel<E, DH><<<pgrid, 256, 0, s>>>(p);
    attn_bwd_dq_kernel<E, DH><<<grid, 256, 0, s>>>(p);
    attn_bwd_dkv_kernel<E, DH><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

// Tensor-core form: the prep kernel (q^, Delta), the forward's log-sum-exp when it was not
// given (the forward attention runs once with its output in dq, which the dq launch then
// overwrites), then the dq and dk/dv launches.
static int launch_bwd_tc(const AttnBwdParams &p, cudaStream_t s) {
    const dim3 pgrid((unsigned)((p.T + 8 * kPrepRows - 1) / (8 * kPrepRows)), (unsigned)(p.B * p.H));
    attn_bwd_prep_kernel<__nv_bfloat16, 128><<<pgrid, 256, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return RAT_ERR_CUDA;
    if (!p.lse_given) {
        AttnSm100Args a;
        std::memset(&a, 0, sizeof(a));
        a.q = p.q; a.k = p.k; a.v = p.v; a.o = p.dq;
        a.B = p.B; a.H = p.H; a.T = p.T; a.d = p.d; a.W = p.W;
        a.pos0 = p.pos0;
        a.rope = p.rope;
        a.scale_log2 = p.scale_log2;
        a.Dh = p.Dh;
        a.n_sink = 0;
        a.lse = p.lse;
        for (int c = 0; c < 64; ++c) a.theta[c] = p.theta[c];
        const int st = launch_attn_sm100(a, s);
        if (st != RAT_OK) return st;
    }
    return launch_attn_bwd_sm100(p, s);
}

int launch_attn_bwd(const AttnBwdParams &p, int dtype, void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (attn_bwd_sm100_supported(p, dtype)) return launch_bwd_tc(p, s);
    if (dtype == RAT_F32) {
        if (p.d == 64) return launch_bwd<float, 64>(p, s);
        if (p.d == 128) return launch_bwd<float, 128>(p, s);
    } else {
        if (p.d == 64) return launch_bwd<__nv_bfloat16, 64>(p, s);
        if (p.d == 128) return launch_bwd<__nv_bfloat16, 128>(p, s);
    }
    return RAT_ERR_UNSUPPORTED;
}

}  // namespace rat
