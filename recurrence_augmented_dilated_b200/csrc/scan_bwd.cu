// scan_bwd.cu -- backward of the prefill recurrence step (gradients of k, v, the gate logits
// and the initial state from the gradients of k~, v~ and of the final state).
//
// The forward step ("RAT+ Deep Dive", section 2.1) is h_t = g_t h_{t-1} + (1 - g_t) x_t per
// channel, for x = k and x = v with one gate g = sigmoid(a), k~ = RoPE(h^k), v~ = h^v.  Its
// reverse-mode derivative runs a linear recurrence backwards in time:
//     mu_t = e_t + g_{t+1} mu_{t+1},   mu_{T-1} = e_{T-1} + dL/dh_{T-1},
// with e^k_t = RoPE_t^T(dk~_t) (the transposed rotation) and e^v_t = dv~_t; then
//     dk_t = (1 - g_t) mu^k_t,   dv_t = (1 - g_t) mu^v_t,
//     da_t = g_t (1 - g_t) [ mu^k_t (h^k_{t-1} - k_t) + mu^v_t (h^v_{t-1} - v_t) ],
//     dh0  = g_0 mu_0,
// where h_{t-1} comes from the forward outputs (h^k = RoPE^T(k~), h^v = v~; h_{-1} = h0).
//
// The backward recurrence is affine in mu, so it is a scan like the forward one, run from the
// end.  Three launches over chunks of 64 rows of one (b, h):
//   reduce : per chunk, the composed map mu_{after chunk} -> mu_{first row} as (A, B);
//   carry  : per (b, h, channel), the chunks' maps composed from the last chunk down, giving the
//            gradient entering each chunk from the right, and dh0;
//   output : per chunk, the recurrence rerun backwards from its carry, writing dk, dv, da.
// Within a chunk a group of d/4 lanes walks the rows one by one (lane l holds the channel
// pairs (2l, 2l+1) and (2l + d/2, 2l+1 + d/2), the RoPE partners), loading U rows at a time.
// No CTA waits for another.  HBM traffic: the reduce pass reads a, dk~, dv~ (3 N elements),
// the output pass reads seven tensors and writes three (10 N), against the 10 N minimum.
//
// The chunk-local form (RESET; RAT's recurrence restarted before every absolute position that
// is a multiple of L) cuts both recurrences at block starts: no gradient passes from a block
// start t to t - 1 (the factor g_t of mu_{t-1} becomes 0, so a chunk map composed across a
// start has A = 0), the state entering a block start is 0 in da, and h0 gets a gradient only
// when row 0 is not a block start.
#include "common.cuh"

namespace rat {

namespace {

template <typename E, int DH>
struct BwdCfg {
    static constexpr int LPR = DH / 4;                 // lanes per row
    static constexpr int SPW = 32 / LPR;               // chunk streams per warp
    static constexpr int ROWB = DH * (int)sizeof(E);
    static constexpr int HALFB = ROWB / 2;
    static constexpr int U = sizeof(E) == 2 ? 3 : 2;   // rows loaded together (output pass)
    static constexpr int UR = sizeof(E) == 2 ? 4 : 2;  // rows loaded together (reduce pass)
    static constexpr int THREADS = 256;
    static constexpr int SPB = THREADS / 32 * SPW;     // chunk streams per CTA
};

// (cos, sin) of (pos0 + t) theta for this lane's two frequencies 2l, 2l+1
template <int DH>
RAT_DEVICE void lane_angle(const RecurBwdParams &p, int cl, long long t, f2_t &c, f2_t &s) {
    float c2[2], s2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int f = 2 * cl + u;
        const long long pos = p.pos0 + t;
        if (p.rope_f32) rope_cs_f32((int)pos, p.theta_f[f], c2[u], s2[u]);
        else rope_cs(pos, p.theta[f], c2[u], s2[u]);
    }
    c = f2(c2[0], c2[1]);
    s = f2(s2[0], s2[1]);
}

// the transposed rotation of a lane's pairs: (x1, x2) -> (x1 c + x2 s, x2 c - x1 s)
RAT_DEVICE void rot_t(const f2_t *y, f2_t c, f2_t s, f2_t *x) {
    const f2_t ns = f2_mul(s, f2(-1.f, -1.f));
    x[0] = f2_fma(y[1], s, f2_mul(y[0], c));
    x[1] = f2_fma(y[0], ns, f2_mul(y[1], c));
}

// does a block of the chunk-local form start at row t?
RAT_DEVICE bool block_start(const RecurBwdParams &p, long long t) { return (p.pos0 + t) % p.reset == 0; }

// one step back in position: angle - theta
RAT_DEVICE void step_back(f2_t &c, f2_t &s, f2_t sc, f2_t ss) {
    const f2_t ns = f2_mul(ss, f2(-1.f, -1.f));
    const f2_t nc = f2_fma(s, ss, f2_mul(c, sc));
    s = f2_fma(c, ns, f2_mul(s, sc));
    c = nc;
}

}  // namespace

template <typename E, int DH, bool RESET>
__global__ void __launch_bounds__(BwdCfg<E, DH>::THREADS) bwd_reduce_kernel(const __grid_constant__ RecurBwdParams p) {
    using C = BwdCfg<E, DH>;
    constexpr int NP = 2, U = C::UR;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cl = lane % C::LPR;
    const long long stream = ((long long)blockIdx.x * (C::THREADS / 32) + warp) * C::SPW + lane / C::LPR;
    if (stream >= (long long)p.BH * p.nch) return;
    const int bh = (int)(stream / p.nch), c = (int)(stream % p.nch);
    const int t0 = c * kBwdRows, t1 = min(t0 + kBwdRows, p.T) - 1;
    const f2_t kOne2 = f2(1.f, 1.f), kZero2 = f2(0.f, 0.f);
    const uint8_t *ga = static_cast<const uint8_t *>(p.a) + (size_t)bh * p.T * C::ROWB;
    const uint8_t *gk = static_cast<const uint8_t *>(p.dyk) + (size_t)bh * p.T * C::ROWB;
    const uint8_t *gv = static_cast<const uint8_t *>(p.dyv) + (size_t)bh * p.T * C::ROWB;

    f2_t gnext[NP] = {kOne2, kOne2};             // g_{t+1}; 1 after the last row
    if (t1 + 1 < p.T) {
        f2_t xa[NP];
        Lane<E>::template load<C::HALFB>(ga + (size_t)(t1 + 1) * C::ROWB, cl, xa);
        gnext[0] = forget_gate2(xa[0]);
        gnext[1] = forget_gate2(xa[1]);
        if (RESET && block_start(p, t1 + 1)) gnext[0] = gnext[1] = kZero2;   // nothing passes a start
    }
    f2_t rc = kOne2, rs = kZero2, sc = kOne2, ss = kZero2;
    if (p.rope) {
        lane_angle<DH>(p, cl, t1, rc, rs);
        sc = f2(p.step_cos[2 * cl], p.step_cos[2 * cl + 1]);
        ss = f2(p.step_sin[2 * cl], p.step_sin[2 * cl + 1]);
    }
    f2_t A[NP] = {kOne2, kOne2}, Bk[NP] = {kZero2, kZero2}, Bv[NP] = {kZero2, kZero2};
    for (int tb = t1; tb >= t0; tb -= U) {
        f2_t xa[U][NP], yk[U][NP], yv[U][NP];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = max(tb - u, t0);             // rows below t0 are not used
            Lane<E>::template load<C::HALFB>(ga + (size_t)t * C::ROWB, cl, xa[u]);
            Lane<E>::template load<C::HALFB>(gk + (size_t)t * C::ROWB, cl, yk[u]);
            Lane<E>::template load<C::HALFB>(gv + (size_t)t * C::ROWB, cl, yv[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (tb - u < t0) break;
            f2_t ek[NP] = {yk[u][0], yk[u][1]};
            if (p.rope) {
                rot_t(yk[u], rc, rs, ek);
                step_back(rc, rs, sc, ss);
            }
            const bool start = RESET && block_start(p, tb - u);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                A[q] = f2_mul(gnext[q], A[q]);
                Bk[q] = f2_fma(gnext[q], Bk[q], ek[q]);
                Bv[q] = f2_fma(gnext[q], Bv[q], yv[u][q]);
                gnext[q] = start ? kZero2 : forget_gate2(xa[u][q]);
            }
        }
    }
    float *o = p.agg + (size_t)stream * 3 * DH;
    const int chq[NP] = {2 * cl, 2 * cl + DH / 2};
#pragma unroll
    for (int q = 0; q < NP; ++q) {
        *reinterpret_cast<float2 *>(o + chq[q]) = make_float2(f2lo(A[q]), f2hi(A[q]));
        *reinterpret_cast<float2 *>(o + DH + chq[q]) = make_float2(f2lo(Bk[q]), f2hi(Bk[q]));
        *reinterpret_cast<float2 *>(o + 2 * DH + chq[q]) = make_float2(f2lo(Bv[q]), f2hi(Bv[q]));
    }
}

// one thread per (b, h, channel): compose the chunks' maps from the last chunk down
template <typename E>
__global__ void __launch_bounds__(128) bwd_carry_kernel(const __grid_constant__ RecurBwdParams p) {
    const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (id >= (long long)p.BH * p.d) return;
    const int bh = (int)(id / p.d), ch = (int)(id % p.d);
    float ck = p.dhTk ? p.dhTk[id] : 0.f, cv = p.dhTv ? p.dhTv[id] : 0.f;
    constexpr int G = 8;                               // chunks whose loads are issued together
    for (int cb = p.nch - 1; cb >= 0; cb -= G) {
        float a[G], bk[G], bv[G];
#pragma unroll
        for (int u = 0; u < G; ++u) {
            const int c = max(cb - u, 0);
            const float *o = p.agg + ((size_t)bh * p.nch + c) * 3 * p.d + ch;
            a[u] = o[0];
            bk[u] = o[p.d];
            bv[u] = o[2 * p.d];
        }
#pragma unroll
        for (int u = 0; u < G; ++u) {
            const int c = cb - u;
            if (c < 0) break;
            float *w = p.carry + ((size_t)bh * p.nch + c) * 2 * p.d + ch;
            w[0] = ck;
            w[p.d] = cv;
            ck = fmaf(a[u], ck, bk[u]);
            cv = fmaf(a[u], cv, bv[u]);
        }
    }
    // ck, cv are now mu_0: dh0 = g_0 mu_0 (0 when row 0 starts a block: h0 is not used)
    if (p.reset > 0 && p.pos0 % p.reset == 0) {
        if (p.dh0k) p.dh0k[id] = 0.f;
        if (p.dh0v) p.dh0v[id] = 0.f;
    } else if (p.dh0k || p.dh0v) {
        float a0;
        const E *ar = static_cast<const E *>(p.a) + (size_t)bh * p.T * p.d + ch;
        if constexpr (sizeof(E) == 2) a0 = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(ar));
        else a0 = *reinterpret_cast<const float *>(ar);
        float g, omg;
        forget_gate(a0, g, omg);
        if (p.dh0k) p.dh0k[id] = g * ck;
        if (p.dh0v) p.dh0v[id] = g * cv;
    }
}

template <typename E, int DH, bool RESET>
__global__ void __launch_bounds__(BwdCfg<E, DH>::THREADS, 2) bwd_out_kernel(const __grid_constant__ RecurBwdParams p) {
    using C = BwdCfg<E, DH>;
    constexpr int NP = 2, U = C::U;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cl = lane % C::LPR;
    const long long stream = ((long long)blockIdx.x * (C::THREADS / 32) + warp) * C::SPW + lane / C::LPR;
    if (stream >= (long long)p.BH * p.nch) return;
    const int bh = (int)(stream / p.nch), c = (int)(stream % p.nch);
    const int t0 = c * kBwdRows, t1 = min(t0 + kBwdRows, p.T) - 1;
    const f2_t kOne2 = f2(1.f, 1.f), kZero2 = f2(0.f, 0.f);
    const size_t base = (size_t)bh * p.T * C::ROWB;
    const uint8_t *ga = static_cast<const uint8_t *>(p.a) + base;
    const uint8_t *gxk = static_cast<const uint8_t *>(p.k) + base;
    const uint8_t *gxv = static_cast<const uint8_t *>(p.v) + base;
    const uint8_t *ghk = static_cast<const uint8_t *>(p.yk) + base;
    const uint8_t *ghv = static_cast<const uint8_t *>(p.yv) + base;
    const uint8_t *gdk = static_cast<const uint8_t *>(p.dyk) + base;
    const uint8_t *gdv = static_cast<const uint8_t *>(p.dyv) + base;
    uint8_t *odk = static_cast<uint8_t *>(p.dk) + base;
    uint8_t *odv = static_cast<uint8_t *>(p.dv) + base;
    uint8_t *oda = static_cast<uint8_t *>(p.da) + base;
    const int chq[NP] = {2 * cl, 2 * cl + DH / 2};

    f2_t muk[NP], muv[NP];
    {
        const float *w = p.carry + (size_t)stream * 2 * DH;
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            muk[q] = f2(w[chq[q]], w[chq[q] + 1]);
            muv[q] = f2(w[DH + chq[q]], w[DH + chq[q] + 1]);
        }
    }
    f2_t gnext[NP] = {kOne2, kOne2};
    if (t1 + 1 < p.T) {
        f2_t xa[NP];
        Lane<E>::template load<C::HALFB>(ga + (size_t)(t1 + 1) * C::ROWB, cl, xa);
        gnext[0] = forget_gate2(xa[0]);
        gnext[1] = forget_gate2(xa[1]);
        if (RESET && block_start(p, t1 + 1)) gnext[0] = gnext[1] = kZero2;
    }
    // rotation at t (for dk~_t) and at t - 1 (for k~_{t-1})
    f2_t rc = kOne2, rs = kZero2, pc = kOne2, ps = kZero2, sc = kOne2, ss = kZero2;
    if (p.rope) {
        lane_angle<DH>(p, cl, t1, rc, rs);
        sc = f2(p.step_cos[2 * cl], p.step_cos[2 * cl + 1]);
        ss = f2(p.step_sin[2 * cl], p.step_sin[2 * cl + 1]);
        pc = rc;
        ps = rs;
        step_back(pc, ps, sc, ss);
    }
    f2_t h0k[NP] = {kZero2, kZero2}, h0v[NP] = {kZero2, kZero2};
    if (t0 == 0) {
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            const size_t o = (size_t)bh * DH + chq[q];
            if (p.h0k) h0k[q] = f2(p.h0k[o], p.h0k[o + 1]);
            if (p.h0v) h0v[q] = f2(p.h0v[o], p.h0v[o + 1]);
        }
    }
    for (int tb = t1; tb >= t0; tb -= U) {
        f2_t xa[U][NP], xk[U][NP], xv[U][NP], hk[U][NP], hv[U][NP], dk[U][NP], dv[U][NP];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = max(tb - u, t0);
            const int tp = max(t - 1, 0);              // row 0's predecessor is h0 (set below)
            Lane<E>::template load<C::HALFB>(ga + (size_t)t * C::ROWB, cl, xa[u]);
            Lane<E>::template load<C::HALFB>(gxk + (size_t)t * C::ROWB, cl, xk[u]);
            Lane<E>::template load<C::HALFB>(gxv + (size_t)t * C::ROWB, cl, xv[u]);
            Lane<E>::template load<C::HALFB>(ghk + (size_t)tp * C::ROWB, cl, hk[u]);
            Lane<E>::template load<C::HALFB>(ghv + (size_t)tp * C::ROWB, cl, hv[u]);
            Lane<E>::template load<C::HALFB>(gdk + (size_t)t * C::ROWB, cl, dk[u]);
            Lane<E>::template load<C::HALFB>(gdv + (size_t)t * C::ROWB, cl, dv[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = tb - u;
            if (t < t0) break;
            f2_t ek[NP] = {dk[u][0], dk[u][1]}, hpk[NP] = {hk[u][0], hk[u][1]};
            if (p.rope) {
                rot_t(dk[u], rc, rs, ek);
                rot_t(hk[u], pc, ps, hpk);
                rc = pc;
                rs = ps;
                step_back(pc, ps, sc, ss);
            }
            f2_t hpv[NP] = {hv[u][0], hv[u][1]};
            if (t == 0) {
#pragma unroll
                for (int q = 0; q < NP; ++q) { hpk[q] = h0k[q]; hpv[q] = h0v[q]; }
            }
            const bool start = RESET && block_start(p, t);
            if (start) {                               // the state entering a block start is 0
#pragma unroll
                for (int q = 0; q < NP; ++q) { hpk[q] = kZero2; hpv[q] = kZero2; }
            }
            f2_t ok[NP], ov[NP], oa[NP];
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                muk[q] = f2_fma(gnext[q], muk[q], ek[q]);
                muv[q] = f2_fma(gnext[q], muv[q], dv[u][q]);
                const f2_t g = forget_gate2(xa[u][q]);
                const f2_t og = gate_complement2(g);
                ok[q] = f2_mul(og, muk[q]);
                ov[q] = f2_mul(og, muv[q]);
                const f2_t sk = f2_fma(xk[u][q], f2(-1.f, -1.f), hpk[q]);     // h_{t-1} - x_t
                const f2_t sv = f2_fma(xv[u][q], f2(-1.f, -1.f), hpv[q]);
                oa[q] = f2_mul(f2_mul(g, og), f2_fma(muk[q], sk, f2_mul(muv[q], sv)));
                gnext[q] = start ? kZero2 : g;
            }
            const size_t o = (size_t)t * C::ROWB;
            Lane<E>::template store<C::HALFB>(odk + o, cl, ok);
            Lane<E>::template store<C::HALFB>(odv + o, cl, ov);
            Lane<E>::template store<C::HALFB>(oda + o, cl, oa);
        }
    }
}

size_t recur_bwd_workspace_bytes(int BH, int T, int d) {
    const size_t nch = ((size_t)T + kBwdRows - 1) / kBwdRows;
    return sizeof(WsHeader) + align256((size_t)BH * nch * 3 * d * 4) + align256((size_t)BH * nch * 2 * d * 4);
}

template <typename E, int DH>
static int launch_bwd_one(const RecurBwdParams &p, cudaStream_t s) {
    using C = BwdCfg<E, DH>;
    const long long streams = (long long)p.BH * p.nch;
    const long long grid = (streams + C::SPB - 1) / C::SPB;
    if (grid > 0x7fffffffll) return RAT_ERR_UNSUPPORTED;
    const long long n = (long long)p.BH * p.d;
    if (p.reset > 0) {
        bwd_reduce_kernel<E, DH, true><<<(unsigned)grid, C::THREADS, 0, s>>>(p);
        bwd_carry_kernel<E><<<(unsigned)((n + 127) / 128), 128, 0, s>>>(p);
        bwd_out_kernel<E, DH, true><<<(unsigned)grid, C::THREADS, 0, s>>>(p);
    } else {
        bwd_reduce_kernel<E, DH, false><<<(unsigned)grid, C::THREADS, 0, s>>>(p);
        bwd_carry_kernel<E><<<(unsigned)((n + 127) / 128), 128, 0, s>>>(p);
        bwd_out_kernel<E, DH, false><<<(unsigned)grid, C::THREADS, 0, s>>>(p);
    }
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

int launch_recur_bwd(const RecurBwdParams &p, int dtype, void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == RAT_F32) {
        if (p.d == 64) return launch_bwd_one<float, 64>(p, s);
        if (p.d == 128) return launch_bwd_one<float, 128>(p, s);
    } else {
        if (p.d == 64) return launch_bwd_one<__nv_bfloat16, 64>(p, s);
        if (p.d == 128) return launch_bwd_one<__nv_bfloat16, 128>(p, s);
    }
    return RAT_ERR_UNSUPPORTED;
}

}  // namespace rat
