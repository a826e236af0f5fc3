// window.cu -- fixed-window forget-gate recurrence over keys and values (prefill).
//
// "RAT+ Deep Dive", section 2.1: RAT+ gives every token a recurrence window of a fixed L* = 64
// tokens, whatever the dilation.  Read as: the state at t is the recurrence h <- g h + (1-g) x
// (g = sigmoid(logit), per channel, x = k and x = v) restarted from zero at t - Lw + 1,
//     y_t = sum_{s = t-Lw+1}^{t} (prod_{r = s+1}^{t} g_r) (1 - g_s) x_s,     Lw = 64.
//
// Segmented form.  Cut the rows into blocks of Lw aligned at row 0.  For t = c Lw + j (row j
// of block c) the window is the tail of block c-1 from its row j + 1 followed by the head of
// block c up to t, so
//     y_t = F_c(t) + P_c(t) U_{c-1}(j + 1),
//   F_c(t)   : the recurrence from zero at the first row of block c, at t;
//   P_c(t)   : the product of block c's gates up to t;
//   U_c(i)   : the recurrence from zero at row i of block c, at the block's last row
//              (U_c(Lw) = 0), kept in registers for block c + 1.  Since the whole block's
//              recurrence E_c splits at row j into Pa_c(j) F_c(j) + U_c(j + 1), with Pa_c(j) the
//              product of the gates after row j, U comes out of the same forward pass as
//              U_c(j + 1) = E_c - Pa_c(j) F_c(j).  Both terms are sums over this block's rows
//              with weights that sum to at most 1, so the difference is exact to a few units in
//              the last place of the block's largest input; no state older than one block is
//              ever subtracted (subtracting the decayed full-sequence state instead would carry
//              the rounding of the whole history).
// No CTA waits for another: the flattened (b, h, block) sequence is cut into one contiguous
// range per CTA, walked in order; the block before a range (or the history rows before row 0)
// is read once more to form its U.
//
// Lane layout as in the full-sequence scan: lane l holds the channel pairs (2l, 2l+1) and
// (2l + d/2, 2l+1 + d/2), the rotate-half RoPE partners.  The 512 threads of a CTA cover one
// block: d/4 lanes per row and 512/(d/4) segments of R consecutive rows (R = 4 for d = 128,
// 2 for d = 64).  Per block: a forward pass over each segment's rows forms its aggregate
// (A = prod g, B = sum ...); one thread per channel combines them through shared memory into
// each segment's carry (exclusive prefix), the block total and the gate product of the later
// segments; a second forward pass from the carry writes the outputs and U.  Blocks stream through a ring of shared-memory stages filled by bulk copies
// (cp.async.bulk) two blocks ahead.  HBM traffic: 3 reads + 2 writes per element, plus one
// extra block per range.
#include "common.cuh"

namespace rat {

namespace {

template <typename E, int DH>
struct WinCfg {
    static constexpr int EB = sizeof(E);
    static constexpr int LW = kWindowRows;              // window = block rows
    static constexpr int THREADS = 512;
    static constexpr int LPR = DH / 4;                  // lanes per row
    static constexpr int SEGS = THREADS / LPR;          // row segments per block
    static constexpr int R = LW / SEGS;                 // rows per segment
    static constexpr int ROWB = DH * EB;
    static constexpr int HALFB = ROWB / 2;
    static constexpr int TILEB = LW * ROWB;             // one tensor of one block
    static constexpr int STAGEB = 3 * TILEB;            // a, k, v
    // [SEGS + 1][3][DH] aggregates -> exclusive prefixes of Bk, Bv (+ block totals), [SEGS][DH]
    // suffix gate products, [SEGS][DH] prefix gate products
    static constexpr int XB = (SEGS + 1) * 3 * DH * 4 + 2 * SEGS * DH * 4;
    static constexpr int FIT = (200 * 1024 - XB) / STAGEB;
    static constexpr int NST = FIT >= 3 ? 3 : (FIT >= 1 ? FIT : 1);   // stages in the ring
    static constexpr int SMEM = NST * STAGEB + XB;
    static_assert(R * SEGS == LW && R >= 1, "whole segments per block");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// The items a CTA walks: for each block of its range, first (when needed) the block before it
// -- only to form U -- then the block itself.  Producer and consumers each step through the
// same sequence with their own cursor.
struct Cursor {
    long long f;          // next flattened block index
    int bh, c;            // its slice and block
    bool prep_done;       // the extra block before f has been returned
};
struct Item {
    int bh, c;            // c = -1: the history rows before row 0
    bool prep;            // true: only U is formed
};

RAT_DEVICE Cursor cursor_at(long long f, int nblk) {
    Cursor cur;
    cur.f = f;
    cur.bh = (int)(f / nblk);
    cur.c = (int)(f % nblk);
    cur.prep_done = false;
    return cur;
}

RAT_DEVICE bool next_item(Cursor &cur, long long f0, long long f1, int nblk, bool has_prev,
                          Item &it) {
    if (cur.f >= f1) return false;
    it.bh = cur.bh;
    const bool need = (cur.f == f0 && cur.c > 0) || (cur.c == 0 && has_prev);
    if (need && !cur.prep_done) {
        it.c = cur.c - 1;
        it.prep = true;
        cur.prep_done = true;
        return true;
    }
    it.c = cur.c;
    it.prep = false;
    cur.prep_done = false;
    ++cur.f;
    if (++cur.c == nblk) {
        cur.c = 0;
        ++cur.bh;
    }
    return true;
}

}  // namespace

template <typename E, int DH>
__global__ void __launch_bounds__(WinCfg<E, DH>::THREADS, 1)
window_kernel(const __grid_constant__ WindowParams p) {
    using C = WinCfg<E, DH>;
    constexpr int LPR = C::LPR, R = C::R, HALF = DH / 2, NP = 2;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bar[C::NST];
    __shared__ float s_theta_f[HALF], s_step_c[HALF], s_step_s[HALF];
    __shared__ double s_theta[HALF];

    const int tid = threadIdx.x;
    const int seg = tid / LPR, cl = tid % LPR;
    const int chq[NP] = {2 * cl, 2 * cl + HALF};                // first channel of each pair
    float *X = reinterpret_cast<float *>(smem + C::NST * C::STAGEB);   // [SEGS + 1][3][DH]
    float *S = X + (C::SEGS + 1) * 3 * DH;                            // [SEGS][DH]
    float *Pt = S + C::SEGS * DH;                                     // [SEGS][DH]
    const long long total = (long long)p.BH * p.nblk;
    const long long f0 = total * blockIdx.x / gridDim.x;
    const long long f1 = total * (blockIdx.x + 1) / gridDim.x;
    const bool has_prev = p.pk != nullptr;
    const f2_t kOne2 = f2(1.f, 1.f), kZero2 = f2(0.f, 0.f), kNegOne2 = f2(-1.f, -1.f);

    // three bulk copies (a, k, v) of one item into stage st (thread 0)
    auto load_item = [&](const Item &it, int st) {
        const uint8_t *ga, *gk, *gv;
        int rows;
        if (it.c < 0) {
            const size_t o = (size_t)it.bh * C::LW * C::ROWB;
            ga = static_cast<const uint8_t *>(p.pa) + o;
            gk = static_cast<const uint8_t *>(p.pk) + o;
            gv = static_cast<const uint8_t *>(p.pv) + o;
            rows = C::LW;
        } else {
            rows = min(C::LW, p.T - it.c * C::LW);
            const size_t o = ((size_t)it.bh * p.T + (size_t)it.c * C::LW) * C::ROWB;
            ga = static_cast<const uint8_t *>(p.a) + o;
            gk = static_cast<const uint8_t *>(p.k) + o;
            gv = static_cast<const uint8_t *>(p.v) + o;
        }
        const uint32_t bytes = (uint32_t)rows * C::ROWB;
        uint8_t *s = smem + st * C::STAGEB;
        mbar_arrive_expect_tx(&bar[st], 3 * bytes);
        bulk_g2s(s, ga, bytes, &bar[st]);
        bulk_g2s(s + C::TILEB, gk, bytes, &bar[st]);
        bulk_g2s(s + 2 * C::TILEB, gv, bytes, &bar[st]);
    };

    if (tid < HALF) {
        s_theta_f[tid] = p.theta_f[tid];
        s_theta[tid] = p.theta[tid];
        s_step_c[tid] = p.step_cos[tid];
        s_step_s[tid] = p.step_sin[tid];
    }
    if (tid == 0) {
        for (int s = 0; s < C::NST; ++s) mbar_init(&bar[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    Cursor pc = cursor_at(f0, p.nblk);    // producer cursor, NST - 1 items ahead (thread 0)
    if (tid == 0) {
        for (int s = 0; s < C::NST - 1; ++s) {
            Item nx;
            if (!next_item(pc, f0, f1, p.nblk, has_prev, nx)) break;
            load_item(nx, s);
        }
    }

    f2_t Uk[R][NP], Uv[R][NP];            // U of the block before the current one, my rows
    int u_bh = -1, u_c = -2;              // the block those U belong to
    bool dead = false;                    // a copy never arrived: skip the rest (error recorded)
    Cursor cc = cursor_at(f0, p.nblk);
    Item it;
    for (int k = 0; next_item(cc, f0, f1, p.nblk, has_prev, it); ++k) {
        const int st = k % C::NST;
        if (tid == 0 && !dead) {          // refill the stage the previous item released
            Item nx;
            if (next_item(pc, f0, f1, p.nblk, has_prev, nx)) load_item(nx, (k + C::NST - 1) % C::NST);
        }
        if (!dead && !mbar_wait_bounded(&bar[st], (uint32_t)(k / C::NST) & 1u, p.hdr, 0x300u))
            dead = true;
        const int rows = it.c < 0 ? C::LW : min(C::LW, p.T - it.c * C::LW);
        const uint8_t *sa = smem + st * C::STAGEB, *sk = sa + C::TILEB, *sv = sa + 2 * C::TILEB;

        // ---- forward pass over my R rows: gates (kept) and the segment aggregate from zero
        f2_t G[R][NP];
        f2_t A[NP] = {kOne2, kOne2}, Bk[NP] = {kZero2, kZero2}, Bv[NP] = {kZero2, kZero2};
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = seg * R + i;
            const int off = (r < rows ? r : rows - 1) * C::ROWB;
            f2_t xa[NP], xk[NP], xv[NP];
            Lane<E>::template load<C::HALFB>(sa + off, cl, xa);
            Lane<E>::template load<C::HALFB>(sk + off, cl, xk);
            Lane<E>::template load<C::HALFB>(sv + off, cl, xv);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                G[i][q] = r < rows ? forget_gate2(xa[q]) : kOne2;     // past the end: identity
                const f2_t og = gate_complement2(G[i][q]);
                A[q] = f2_mul(A[q], G[i][q]);
                Bk[q] = f2_fma(G[i][q], Bk[q], f2_mul(og, xk[q]));
                Bv[q] = f2_fma(G[i][q], Bv[q], f2_mul(og, xv[q]));
            }
        }
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            float *x = X + seg * 3 * DH + chq[q];
            x[0] = f2lo(A[q]);           x[1] = f2hi(A[q]);
            x[DH] = f2lo(Bk[q]);         x[DH + 1] = f2hi(Bk[q]);
            x[2 * DH] = f2lo(Bv[q]);     x[2 * DH + 1] = f2hi(Bv[q]);
        }
        __syncthreads();

        // ---- three walks over the segments, one thread per channel each: the product of the
        // gates of the segments after s into S; the gates before s into Pt with the exclusive
        // prefix of Bk over X in place; the exclusive prefix of Bv; block totals in X[SEGS]
        // (A is only read, so the walks run side by side)
        if (tid < 3 * DH) {
            const int w = tid / DH, ch = tid % DH;
            constexpr int GS = DH == 128 ? 8 : 4;      // segments loaded ahead of the chain
            if (w == 2) {
                float sA = 1.f;
#pragma unroll 1
                for (int g0 = C::SEGS - GS; g0 >= 0; g0 -= GS) {
                    float xa[GS];
#pragma unroll
                    for (int u = 0; u < GS; ++u) xa[u] = X[(g0 + u) * 3 * DH + ch];
#pragma unroll
                    for (int u = GS - 1; u >= 0; --u) {
                        S[(g0 + u) * DH + ch] = sA;
                        sA *= xa[u];
                    }
                }
            } else {
                const int off = w ? 2 * DH : DH;       // Bk or Bv
                float pA = 1.f, pB = 0.f;
#pragma unroll 1
                for (int g0 = 0; g0 < C::SEGS; g0 += GS) {
                    float xa[GS], xb[GS];
#pragma unroll
                    for (int u = 0; u < GS; ++u) {
                        const float *x = X + (g0 + u) * 3 * DH + ch;
                        xa[u] = x[0];
                        xb[u] = x[off];
                    }
#pragma unroll
                    for (int u = 0; u < GS; ++u) {
                        if (w == 0) Pt[(g0 + u) * DH + ch] = pA;
                        X[(g0 + u) * 3 * DH + ch + off] = pB;
                        pB = fmaf(xa[u], pB, xb[u]);
                        pA *= xa[u];
                    }
                }
                X[C::SEGS * 3 * DH + ch + off] = pB;
            }
        }
        __syncthreads();

        // ---- forward over my rows again from the segment's carry: F and P, the outputs
        // y = F + P U(j + 1) (k~ rotated), and U of this block for the next one,
        //     U(j + 1) = E - Pa(j) F(j),
        // E = the block total, Pa(j) = the product of the block's gates after row j.  E and
        // Pa F are both sums over this block's rows with weights summing to at most 1, so the
        // difference is exact to a few units of the block's largest input.
        const bool needU = it.c + 1 < p.nblk;           // a next block of this slice exists
        if (!it.prep && !(u_bh == it.bh && u_c == it.c - 1)) {
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int q = 0; q < NP; ++q) { Uk[i][q] = kZero2; Uv[i][q] = kZero2; }
        }
        f2_t Fk[NP], Fv[NP], Pp[NP], Ek[NP], Ev[NP], npa[R][NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            const float *x = X + seg * 3 * DH + chq[q];
            Pp[q] = f2(Pt[seg * DH + chq[q]], Pt[seg * DH + chq[q] + 1]);
            Fk[q] = f2(x[DH], x[DH + 1]);
            Fv[q] = f2(x[2 * DH], x[2 * DH + 1]);
            const float *e = X + C::SEGS * 3 * DH + chq[q];
            Ek[q] = f2(e[DH], e[DH + 1]);
            Ev[q] = f2(e[2 * DH], e[2 * DH + 1]);
            const float *o = S + seg * DH + chq[q];
            npa[R - 1][q] = f2(-o[0], -o[1]);           // minus the gates after my last row
#pragma unroll
            for (int i = R - 2; i >= 0; --i) npa[i][q] = f2_mul(npa[i + 1][q], G[i + 1][q]);
        }
        f2_t rc = kOne2, rs = kZero2, sc = kOne2, ss = kZero2, nss = kZero2;
        if (p.rope && !it.prep) {
            const long long pos = p.pos0 + (long long)it.c * C::LW + seg * R;
            float c2[2], s2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int f = 2 * cl + u;
                if (p.rope_f32) rope_cs_f32((int)pos, s_theta_f[f], c2[u], s2[u]);
                else rope_cs(pos, s_theta[f], c2[u], s2[u]);
            }
            rc = f2(c2[0], c2[1]);
            rs = f2(s2[0], s2[1]);
            sc = f2(s_step_c[2 * cl], s_step_c[2 * cl + 1]);
            ss = f2(s_step_s[2 * cl], s_step_s[2 * cl + 1]);
            nss = f2(-s_step_s[2 * cl], -s_step_s[2 * cl + 1]);
        }
        uint8_t *yk = static_cast<uint8_t *>(p.yk);
        uint8_t *yv = static_cast<uint8_t *>(p.yv);
        const size_t row0 = (size_t)it.bh * p.T + (size_t)it.c * C::LW;
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = seg * R + i;
            const int off = (r < rows ? r : rows - 1) * C::ROWB;
            f2_t xk[NP], xv[NP], hk[NP], hv[NP];
            Lane<E>::template load<C::HALFB>(sk + off, cl, xk);
            Lane<E>::template load<C::HALFB>(sv + off, cl, xv);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const f2_t og = gate_complement2(G[i][q]);
                Fk[q] = f2_fma(G[i][q], Fk[q], f2_mul(og, xk[q]));
                Fv[q] = f2_fma(G[i][q], Fv[q], f2_mul(og, xv[q]));
                Pp[q] = f2_mul(Pp[q], G[i][q]);
                hk[q] = f2_fma(Pp[q], Uk[i][q], Fk[q]);
                hv[q] = f2_fma(Pp[q], Uv[i][q], Fv[q]);
                Uk[i][q] = f2_fma(npa[i][q], Fk[q], Ek[q]);
                Uv[i][q] = f2_fma(npa[i][q], Fv[q], Ev[q]);
            }
            if (!it.prep) {
                f2_t ok[NP] = {hk[0], hk[1]};
                if (p.rope) {
                    const f2_t nrs = f2_mul(rs, kNegOne2);
                    ok[0] = f2_fma(hk[1], nrs, f2_mul(hk[0], rc));
                    ok[1] = f2_fma(hk[0], rs, f2_mul(hk[1], rc));
                    const f2_t nc = f2_fma(rc, sc, f2_mul(rs, nss));     // advance one position
                    rs = f2_fma(rs, sc, f2_mul(rc, ss));
                    rc = nc;
                }
                if (r < rows && !dead) {
                    const size_t go = (row0 + r) * C::ROWB;
                    Lane<E>::template store<C::HALFB>(yk + go, cl, ok);
                    Lane<E>::template store<C::HALFB>(yv + go, cl, hv);
                }
            }
        }
        if (needU) {
            u_bh = it.bh;
            u_c = it.c;
        }
        __syncthreads();        // the stage and the X / S tables are free for the next item
    }
}

template <typename E, int DH>
static int launch_one(const WindowParams &p, void *stream) {
    using C = WinCfg<E, DH>;
    auto kern = window_kernel<E, DH>;
    static std::atomic<uint64_t> attr_done{0};
    const int st = set_smem_attr(reinterpret_cast<const void *>(kern), C::SMEM, &attr_done);
    if (st != RAT_OK) return st;
    const int sms = current_sm_count();
    if (sms <= 0) return RAT_ERR_CUDA;
    // one CTA per SM, each a contiguous range of blocks (ranges differ by at most one block)
    const long long total = (long long)p.BH * p.nblk;
    const unsigned grid = (unsigned)(total < sms ? total : sms);
    kern<<<grid, C::THREADS, C::SMEM, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

int launch_window(const WindowParams &p, int dtype, void *stream) {
    if (dtype == RAT_F32) {
        if (p.d == 64) return launch_one<float, 64>(p, stream);
        if (p.d == 128) return launch_one<float, 128>(p, stream);
    } else {
        if (p.d == 64) return launch_one<__nv_bfloat16, 64>(p, stream);
        if (p.d == 128) return launch_one<__nv_bfloat16, 128>(p, stream);
    }
    return RAT_ERR_UNSUPPORTED;
}

}  // namespace rat
