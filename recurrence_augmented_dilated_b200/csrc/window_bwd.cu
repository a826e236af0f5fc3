// window_bwd.cu -- backward of the fixed-window recurrence (gradients of k, v, the gate logits
// and of the history rows, from the gradients of k~, v~).
//
// "RAT+ Deep Dive", section 2.1 gives every token a recurrence window of L* = 64 positions.  Read
// as: y_t is the recurrence h <- g h + (1-g) x restarted from zero at t - Lw + 1 (per channel,
// x = k and x = v, one gate g = sigmoid(a)), k~ = RoPE(y^k), v~ = y^v.  With e = dL/dy
// (e^k = RoPE^T(dk~), e^v = dv~) and the rows cut into blocks of Lw aligned at row 0 (block -1:
// the history rows), the output at row j of block c is y = F_c(j) + P_c(j) U_{c-1}(j + 1), where
//   F(j)     the recurrence from zero at the block's first row, at row j     (F(-1) = 0),
//   P(j)     the product of the block's gates up to row j                    (P(-1) = 1),
//   D(j)     the product of the block's gates after row j                    (D(Lw-1) = 1),
//   U(j+1)   = E - D(j) F(j): the recurrence from zero at row j + 1, at the block's last row
//            (E = F(Lw-1), U(Lw) = 0).
// Differentiating that form, the gradients at row j of block c are
//   dx(j) = (1 - g(j)) (mu(j) + D(j) Lam(j)),
//   dg(j) = mu(j) (F(j-1) - x(j)) + P(j-1) rho(j) + D(j) (Y(j-1) - x(j) Lam(j)),
//   dL/da = g (1 - g) (dg^k + dg^v),
// with three reverse / forward sums inside the block
//   mu(j)  = e(j) + g(j+1) mu(j+1),                    mu(Lw) = 0    (through F_c),
//   rho(j) = e(j) U_{c-1}(j+1) + g(j+1) rho(j+1),      rho(Lw) = 0   (through P_c),
//   Y(j)   = g(j) Y(j-1) + (1 - g(j)) x(j) Lam(j),     Y(-1) = 0,
// and one from the next block, through U_c:
//   Lam(j) = sum_{r < j} e_{c+1}(r) P_{c+1}(r)         (0 after the last block).
// Every term is a product of gates of one block, so nothing is divided by a gate and no state
// older than a block is subtracted.
//
// Work split.  Each (b, h) is cut into channel slices (64 channels for bf16, 32 for float32:
// half from the first half of the row and their rotate-half RoPE partners).  The flattened
// ((b, h), block) sequence is cut into contiguous ranges, and each range is walked in order by one
// CTA per slice (one CTA per SM, the slices of a range on neighbouring SMs, so the 128-byte lines
// they share are read from HBM once); U of the block before a range (or the history rows) comes
// from one extra block at its start, and Lam of a range's last block from the next block's a,
// dk~, dv~.  No CTA waits for another.
//
// Per block, 16 segments of 4 rows; a lane holds two channel pairs of its rows (a pair and its
// RoPE partner), so the transposed rotation of dk~ needs nothing from other lanes:
//   1. each lane forms its segment's aggregates: the next block's gate product and its sum of
//      e P (for Lam), this block's gate product, local F, Y driven by the segment's own part of
//      Lam, and the local reverse sums of mu and rho;
//   2. four walks over the 16 segments, one thread per channel each: forwards for k and for v
//      (Lam, P, F, Y entering each segment, and E), backwards for k and for v (D and the mu, rho
//      carries entering from the right);
//   3. each lane finishes its rows: dk, dv, da, and U of this block for the next one (kept in
//      registers, like the next block's gates, which the look-ahead forms once for both uses).
// Data movement: per block the slices of a, dk~, dv~ and of k, v arrive by cp.async in two
// rings (three and two stages), issued three and two blocks ahead; the next block's a, dk~, dv~
// serve as this block's look-ahead and then as the next block's own data.  HBM traffic: five
// reads and three writes per element, plus one block per range.
#include "common.cuh"

namespace rat {

namespace {

template <typename E>
struct WbCfg {
    static constexpr int EB = sizeof(E);
    static constexpr int LW = kWindowRows;            // rows per block = the window
    static constexpr int SW = EB == 2 ? 64 : 32;      // channels per slice: a 128-byte row piece
    static constexpr int HSW = SW / 2;                // first-half channels per slice
    static constexpr int LPR = SW / 4;                // lanes per row, two pairs each
    static constexpr int R = 4;                       // rows per segment
    static constexpr int SEGS = LW / R;
    static constexpr int THREADS = LPR * SEGS;        // 256 (bf16) or 128 (float32)
    static constexpr int ROWB = SW * EB;
    static constexpr int TILEB = LW * ROWB;           // one tensor's slice of one block
    static constexpr int PIECES = TILEB / 16;         // 16-byte copies per tile
    static constexpr int PPT = PIECES / THREADS;      // per thread
    static constexpr int NAGD = 3, NKV = 2;           // ring stages: (a, dk~, dv~) and (k, v)
    static constexpr int AGDB = 3 * TILEB, KVB = 2 * TILEB;
    static constexpr int TABB = SEGS * SW * 4;        // one [SEGS][SW] float table
    static constexpr int NTAB = 15;
    static constexpr int OFF_KV = NAGD * AGDB;
    static constexpr int OFF_TAB = OFF_KV + NKV * KVB;
    static constexpr int OFF_E = OFF_TAB + NTAB * TABB;
    static constexpr int SMEM = OFF_E + 2 * SW * 4;
    static_assert(ROWB == 128 && PPT * THREADS == PIECES, "tile geometry");
    static_assert(SEGS * R == LW && THREADS == 4 * SW, "four walks of one thread per channel");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Per-segment tables [SEGS][SW]: step 1 writes the aggregates, step 2 the carries entering each
// segment, in place where one walk alone reads the aggregate (A and AN are read by several).
enum : int {
    T_AN = 0,    // next block's gate product
    T_KNK, T_KNV,// next block's sum of e P          -> Lam entering the segment (k, v)
    T_A,         // this block's gate product
    T_BFK, T_BFV,// local F                          -> F entering the segment
    T_YPK, T_YPV,// local Y driven by the segment's own part of Lam -> Y entering the segment
    T_BMK, T_BMV,// local reverse mu carry           -> mu carry entering from the right
    T_BRK, T_BRV,// local reverse rho carry          -> rho carry entering from the right
    T_P,         //                                    product of the gates before the segment
    T_D,         //                                    product of the gates after the segment
    T_PN,        //                                    next block: product of its gates before it
};

enum : int { kNone = 0, kPrep = 1, kMain = 2, kTail = 3 };
struct WbItem {
    int kind;     // kPrep: only U of the block; kMain: the block's gradients; kTail: look-ahead data
    int bh;       // (b, h)
    int c;        // block (-1: the history rows)
};
struct WbCursor {
    long long f;  // next flattened (b, h, block) index of the range
    int bh, c;    // that item
    bool prep_done, tail_done;
};

RAT_DEVICE WbCursor wb_cursor(long long f0, int nchain, int cmin) {
    WbCursor cur;
    cur.f = f0;
    cur.bh = (int)(f0 / nchain);
    cur.c = cmin + (int)(f0 - (long long)cur.bh * nchain);
    cur.prep_done = cur.tail_done = false;
    return cur;
}

// The items a CTA walks, in order: for each block of its range (blocks -1 .. nblk-1 of every
// (b, h) when the history rows get gradients, else 0 .. nblk-1), first -- at the range start or
// a (b, h) start, when that block exists -- the block before it (kPrep, for U), then the block
// itself (kMain); after the range, the block after its last one (kTail), if any.
RAT_DEVICE WbItem wb_next(WbCursor &cur, long long f0, long long f1, int nblk, int cmin,
                          bool has_prev) {
    if (cur.f < f1) {
        const int c = cur.c;
        const bool need = (cur.f == f0 || c == cmin) && (c >= 1 || (c == 0 && has_prev));
        if (need && !cur.prep_done) {
            cur.prep_done = true;
            return WbItem{kPrep, cur.bh, c - 1};
        }
        const WbItem it{kMain, cur.bh, c};
        cur.prep_done = false;
        ++cur.f;
        if (++cur.c == nblk) {
            cur.c = cmin;
            ++cur.bh;
        }
        return it;
    }
    if (!cur.tail_done && f1 > f0) {
        cur.tail_done = true;
        if (cur.c != cmin) return WbItem{kTail, cur.bh, cur.c};   // the range ended inside a (b, h)
    }
    return WbItem{kNone, 0, 0};
}

RAT_DEVICE void cp_async16(void *sdst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(smem_u32(sdst)), "l"(gsrc) : "memory");
}
RAT_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
RAT_DEVICE void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
RAT_DEVICE void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// A lane's two channel pairs of one tile row.  Rows whose (index >> 1) is odd hold their two
// 64-byte halves swapped, so the two row groups a warp reads together use different banks.
template <typename E> struct WbLane;
template <> struct WbLane<__nv_bfloat16> {
    static RAT_DEVICE void load(const uint8_t *row, int o0, int o1, int l, f2_t *x) {
        x[0] = f2_from_bf16x2(*reinterpret_cast<const uint32_t *>(row + o0 + 4 * l));
        x[1] = f2_from_bf16x2(*reinterpret_cast<const uint32_t *>(row + o1 + 4 * l));
    }
    static RAT_DEVICE void store(uint8_t *g0, uint8_t *g1, const f2_t *x) {
        *reinterpret_cast<uint32_t *>(g0) = f2_to_bf16x2(x[0]);
        *reinterpret_cast<uint32_t *>(g1) = f2_to_bf16x2(x[1]);
    }
};
template <> struct WbLane<float> {
    static RAT_DEVICE void load(const uint8_t *row, int o0, int o1, int l, f2_t *x) {
        const uint2 a = *reinterpret_cast<const uint2 *>(row + o0 + 8 * l);
        const uint2 b = *reinterpret_cast<const uint2 *>(row + o1 + 8 * l);
        x[0] = f2(__uint_as_float(a.x), __uint_as_float(a.y));
        x[1] = f2(__uint_as_float(b.x), __uint_as_float(b.y));
    }
    static RAT_DEVICE void store(uint8_t *g0, uint8_t *g1, const f2_t *x) {
        *reinterpret_cast<uint2 *>(g0) = make_uint2(__float_as_uint(f2lo(x[0])), __float_as_uint(f2hi(x[0])));
        *reinterpret_cast<uint2 *>(g1) = make_uint2(__float_as_uint(f2lo(x[1])), __float_as_uint(f2hi(x[1])));
    }
};

// the transposed rotation of a lane's pairs: (y1, y2) -> (y1 c + y2 s, y2 c - y1 s)
RAT_DEVICE void rot_t(const f2_t *y, f2_t c, f2_t s, f2_t *x) {
    const f2_t ns = f2_mul(s, f2(-1.f, -1.f));
    x[0] = f2_fma(y[1], s, f2_mul(y[0], c));
    x[1] = f2_fma(y[0], ns, f2_mul(y[1], c));
}

// one step forward in position: angle + theta
RAT_DEVICE void step_fwd(f2_t &c, f2_t &s, f2_t sc, f2_t ss) {
    const f2_t nss = f2_mul(ss, f2(-1.f, -1.f));
    const f2_t nc = f2_fma(s, nss, f2_mul(c, sc));
    s = f2_fma(c, ss, f2_mul(s, sc));
    c = nc;
}

RAT_DEVICE f2_t ld_f2(const float *p) { return *reinterpret_cast<const f2_t *>(p); }
RAT_DEVICE void st_f2(float *p, f2_t v) { *reinterpret_cast<f2_t *>(p) = v; }

}  // namespace

template <typename E>
__global__ void __launch_bounds__(WbCfg<E>::THREADS, 1)
window_bwd_kernel(const __grid_constant__ WindowBwdParams p) {
    using C = WbCfg<E>;
    constexpr int LW = C::LW, SW = C::SW, HSW = C::HSW, LPR = C::LPR, SEGS = C::SEGS, R = C::R;
    constexpr int TS = SEGS * SW;                      // floats per table
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ float s_theta_f[64], s_step_c[64], s_step_s[64], s_step64_c[64], s_step64_s[64];
    __shared__ double s_theta[64];

    const int tid = threadIdx.x;
    const int seg = tid / LPR, cl = tid % LPR;
    const int j0 = seg * R;                            // my rows j0 .. j0 + R - 1 of every block
    const int o0 = (seg & 1) ? 64 : 0, o1 = 64 - o0;   // where my rows keep their two halves
    // CTA b takes slice b mod ns of range b / ns: the ns slices of a range run side by side on
    // neighbouring SMs and read the same 128-byte lines at about the same time
    const int ns = p.d / SW;                           // slices per (b, h)
    const int sl = blockIdx.x % ns;
    const int nranges = gridDim.x / ns, range = blockIdx.x / ns;
    const bool has_prev = p.pk != nullptr;
    const int cmin = p.dpk != nullptr ? -1 : 0;        // the history rows get gradients
    const int nchain = p.nblk - cmin;
    const long long total = (long long)p.BH * nchain;
    const long long f0 = total * range / nranges;
    const long long f1 = total * (range + 1) / nranges;
    const size_t rowstride = (size_t)p.d * C::EB;
    const size_t halfoff = (size_t)(p.d / 2) * C::EB;  // first half -> partner half of a row
    const size_t col = (size_t)sl * HSW * C::EB;       // my slice's first bytes of a row
    const int fq = sl * HSW + 2 * cl;                  // my two RoPE frequencies fq, fq + 1
    float *tab = reinterpret_cast<float *>(smem + C::OFF_TAB);
    float *Etab = reinterpret_cast<float *>(smem + C::OFF_E);   // [2][SW] block totals
    const f2_t kOne2 = f2(1.f, 1.f), kZero2 = f2(0.f, 0.f), kNeg2 = f2(-1.f, -1.f);

    if (tid < 64) {
        s_theta_f[tid] = p.theta_f[tid];
        s_theta[tid] = p.theta[tid];
        s_step_c[tid] = p.step_cos[tid];
        s_step_s[tid] = p.step_sin[tid];
        s_step64_c[tid] = p.step64_cos[tid];
        s_step64_s[tid] = p.step64_sin[tid];
    }

    // copy the slice of rows [0, rows) of one block of a tensor into a tile (rows of odd
    // segment index keep their two halves swapped)
    auto load_tile = [&](uint8_t *tile, const uint8_t *g, int rows) {
#pragma unroll
        for (int u = 0; u < C::PPT; ++u) {
            const int pc = tid + u * C::THREADS;
            const int r = pc >> 3, q = pc & 7;
            if (r < rows) {
                const uint8_t *src = g + (size_t)r * rowstride + (q < 4 ? q * 16 : halfoff + (q - 4) * 16);
                cp_async16(tile + r * C::ROWB + ((q ^ (((r / R) & 1) << 2)) << 4), src);
            }
        }
    };
    // byte address of row 0 of block c of (b, h) = bh of a tensor, my slice (c = -1: history)
    auto block_src = [&](const void *t, const void *hist, int bh, int c) -> const uint8_t * {
        if (c < 0) return static_cast<const uint8_t *>(hist) + (size_t)bh * LW * rowstride + col;
        return static_cast<const uint8_t *>(t) + ((size_t)bh * p.T + (size_t)c * LW) * rowstride + col;
    };
    auto block_rows = [&](int c) { return c < 0 ? LW : min(LW, p.T - c * LW); };
    // a, and dk~ / dv~ when the item needs them, into stage s of the first ring
    auto issue_agd = [&](const WbItem &it, int s) {
        if (it.kind == kNone) return;
        uint8_t *st = smem + s * C::AGDB;
        const int rows = block_rows(it.c);
        load_tile(st, block_src(p.a, p.pa, it.bh, it.c), rows);
        if (it.kind != kPrep && it.c >= 0) {
            load_tile(st + C::TILEB, block_src(p.dyk, nullptr, it.bh, it.c), rows);
            load_tile(st + 2 * C::TILEB, block_src(p.dyv, nullptr, it.bh, it.c), rows);
        }
    };
    auto issue_kv = [&](const WbItem &it, int s) {
        if (it.kind != kPrep && it.kind != kMain) return;
        uint8_t *st = smem + C::OFF_KV + s * C::KVB;
        const int rows = block_rows(it.c);
        load_tile(st, block_src(p.k, p.pk, it.bh, it.c), rows);
        load_tile(st + C::TILEB, block_src(p.v, p.pv, it.bh, it.c), rows);
    };
    // (cos, sin) of this lane's two frequencies at position pos
    auto lane_angle = [&](long long pos, f2_t &c, f2_t &s) {
        float c2[2], s2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (p.rope_f32) rope_cs_f32((int)pos, s_theta_f[fq + u], c2[u], s2[u]);
            else rope_cs(pos, s_theta[fq + u], c2[u], s2[u]);
        }
        c = f2(c2[0], c2[1]);
        s = f2(s2[0], s2[1]);
    };
    f2_t sc = kOne2, ss = kZero2, sc64 = kOne2, ss64 = kZero2;   // rotations by 1 and 64 positions
    // e^k, e^v of my rows of a block from its dk~, dv~ tiles (0 past `rows`); (rc, rs) is the
    // angle of row j0
    auto load_e = [&](const uint8_t *sdk, const uint8_t *sdv, int rows, f2_t rc, f2_t rs,
                      f2_t (&ek)[R][2], f2_t (&ev)[R][2]) {
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int j = j0 + i;
            f2_t yk[2];
            WbLane<E>::load(sdk + j * C::ROWB, o0, o1, cl, yk);
            WbLane<E>::load(sdv + j * C::ROWB, o0, o1, cl, ev[i]);
            if (p.rope) {
                rot_t(yk, rc, rs, ek[i]);
                step_fwd(rc, rs, sc, ss);
            } else {
                ek[i][0] = yk[0];
                ek[i][1] = yk[1];
            }
            if (j >= rows) ek[i][0] = ek[i][1] = ev[i][0] = ev[i][1] = kZero2;
        }
    };

    __syncthreads();
    if (p.rope) {
        sc = f2(s_step_c[fq], s_step_c[fq + 1]);
        ss = f2(s_step_s[fq], s_step_s[fq + 1]);
        sc64 = f2(s_step64_c[fq], s_step64_c[fq + 1]);
        ss64 = f2(s_step64_s[fq], s_step64_s[fq + 1]);
    }
    // prologue: (a, dk~, dv~) of items 0..2 and (k, v) of items 0..1
    WbCursor ca = wb_cursor(f0, nchain, cmin), ck = ca, cc = ca;
    {
        const WbItem a0 = wb_next(ca, f0, f1, p.nblk, cmin, has_prev);
        const WbItem a1 = wb_next(ca, f0, f1, p.nblk, cmin, has_prev);
        const WbItem k0 = wb_next(ck, f0, f1, p.nblk, cmin, has_prev);
        issue_agd(a0, 0);
        issue_kv(k0, 0);
        issue_agd(a1, 1);
        cp_async_commit();
        const WbItem a2 = wb_next(ca, f0, f1, p.nblk, cmin, has_prev);
        const WbItem k1 = wb_next(ck, f0, f1, p.nblk, cmin, has_prev);
        issue_agd(a2, 2);
        issue_kv(k1, 1);
        cp_async_commit();
    }

    f2_t U1k[R][2], U1v[R][2];   // U of the block before, at rows j + 1, for my rows j (k, v)
    f2_t gcar[R][2];             // gates of the block after the last one, from its look-ahead
    int u_bh = -1, u_c = -3, g_bh = -1, g_c = -3;
    for (int it_k = 0;; ++it_k) {
        const WbItem it = wb_next(cc, f0, f1, p.nblk, cmin, has_prev);
        if (it.kind != kPrep && it.kind != kMain) break;
        cp_async_wait_1();
        __syncthreads();

        const bool prep = it.kind == kPrep;
        const int bh = it.bh, c = it.c;
        const int rows = block_rows(c);
        const bool has_next = !prep && c + 1 < p.nblk;
        const bool has_e = !prep && c >= 0;
        const uint8_t *sa = smem + (it_k % C::NAGD) * C::AGDB;
        const uint8_t *sk = smem + C::OFF_KV + (it_k & 1) * C::KVB, *sv = sk + C::TILEB;
        // RoPE angle of row j0 of this block, and of the next one (64 positions on)
        f2_t rc = kOne2, rs = kZero2, nrc = kOne2, nrs = kZero2;
        if (p.rope && (has_e || has_next)) {
            lane_angle(p.pos0 + (long long)c * LW + j0, rc, rs);
            nrc = f2_fma(rs, f2_mul(ss64, kNeg2), f2_mul(rc, sc64));
            nrs = f2_fma(rc, ss64, f2_mul(rs, sc64));
        }
        if (!(u_bh == bh && u_c == c - 1)) {
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int q = 0; q < 2; ++q) U1k[i][q] = U1v[i][q] = kZero2;
        }

        // ---- 1. segment aggregates (the gates of my rows stay in registers until step 3)
        f2_t g[R][2];
        f2_t lk[R][2], lv[R][2];    // Lam's steps inside my segment, sum_{r < i} e'(r) P'(r)
        if (g_bh == bh && g_c == c) {
#pragma unroll
            for (int i = 0; i < R; ++i) { g[i][0] = gcar[i][0]; g[i][1] = gcar[i][1]; }
        } else {
#pragma unroll
            for (int i = 0; i < R; ++i) {
                f2_t xa[2];
                WbLane<E>::load(sa + (j0 + i) * C::ROWB, o0, o1, cl, xa);
#pragma unroll
                for (int q = 0; q < 2; ++q) g[i][q] = j0 + i < rows ? forget_gate2(xa[q]) : kOne2;
            }
        }
        // my rows' x and e (k~ rotated back), from shared memory (again in step 3)
        auto load_xe = [&](f2_t (&xk)[R][2], f2_t (&xv)[R][2], f2_t (&ek)[R][2], f2_t (&ev)[R][2]) {
#pragma unroll
            for (int i = 0; i < R; ++i) {
                WbLane<E>::load(sk + (j0 + i) * C::ROWB, o0, o1, cl, xk[i]);
                WbLane<E>::load(sv + (j0 + i) * C::ROWB, o0, o1, cl, xv[i]);
                if (j0 + i >= rows) xk[i][0] = xk[i][1] = xv[i][0] = xv[i][1] = kZero2;
            }
            if (has_e) {
                load_e(sa + C::TILEB, sa + 2 * C::TILEB, rows, rc, rs, ek, ev);
            } else {
#pragma unroll
                for (int i = 0; i < R; ++i) ek[i][0] = ek[i][1] = ev[i][0] = ev[i][1] = kZero2;
            }
        };
        // look-ahead over the next block: its gates (kept for the next item), its gate product
        // over my rows, and Lam's steps inside my segment
        {
            f2_t xk[R][2], xv[R][2], ek[R][2], ev[R][2];
            load_xe(xk, xv, ek, ev);
            f2_t An[2] = {kOne2, kOne2}, Kk[2] = {kZero2, kZero2}, Kv[2] = {kZero2, kZero2};
            if (has_next) {
                const uint8_t *na = smem + ((it_k + 1) % C::NAGD) * C::AGDB;
                const int nrows = block_rows(c + 1);
                f2_t nek[R][2], nev[R][2];
                load_e(na + C::TILEB, na + 2 * C::TILEB, nrows, nrc, nrs, nek, nev);
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    f2_t xa[2];
                    WbLane<E>::load(na + (j0 + i) * C::ROWB, o0, o1, cl, xa);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const f2_t gn = j0 + i < nrows ? forget_gate2(xa[q]) : kOne2;
                        gcar[i][q] = gn;
                        lk[i][q] = Kk[q];
                        lv[i][q] = Kv[q];
                        An[q] = f2_mul(An[q], gn);
                        Kk[q] = f2_fma(nek[i][q], An[q], Kk[q]);
                        Kv[q] = f2_fma(nev[i][q], An[q], Kv[q]);
                    }
                }
                g_bh = bh;
                g_c = c + 1;
            } else {
#pragma unroll
                for (int i = 0; i < R; ++i) lk[i][0] = lk[i][1] = lv[i][0] = lv[i][1] = kZero2;
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                f2_t A = kOne2, bfk = kZero2, bfv = kZero2, ypk = kZero2, ypv = kZero2;
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    const f2_t og = gate_complement2(g[i][q]);
                    const f2_t uk = f2_mul(og, xk[i][q]), uv = f2_mul(og, xv[i][q]);
                    A = f2_mul(A, g[i][q]);
                    bfk = f2_fma(g[i][q], bfk, uk);
                    bfv = f2_fma(g[i][q], bfv, uv);
                    ypk = f2_fma(g[i][q], ypk, f2_mul(uk, lk[i][q]));
                    ypv = f2_fma(g[i][q], ypv, f2_mul(uv, lv[i][q]));
                }
                // reverse sums from the segment's end: m <- g(j) (s(j) + m)
                f2_t bmk = kZero2, bmv = kZero2, brk = kZero2, brv = kZero2;
#pragma unroll
                for (int i = R - 1; i >= 0; --i) {
                    bmk = f2_mul(g[i][q], f2_add(ek[i][q], bmk));
                    bmv = f2_mul(g[i][q], f2_add(ev[i][q], bmv));
                    brk = f2_mul(g[i][q], f2_fma(ek[i][q], U1k[i][q], brk));
                    brv = f2_mul(g[i][q], f2_fma(ev[i][q], U1v[i][q], brv));
                }
                float *t = tab + seg * SW + (q ? HSW : 0) + 2 * cl;
                st_f2(t + T_AN * TS, An[q]);
                st_f2(t + T_KNK * TS, Kk[q]);
                st_f2(t + T_KNV * TS, Kv[q]);
                st_f2(t + T_A * TS, A);
                st_f2(t + T_BFK * TS, bfk);
                st_f2(t + T_BFV * TS, bfv);
                st_f2(t + T_YPK * TS, ypk);
                st_f2(t + T_YPV * TS, ypv);
                st_f2(t + T_BMK * TS, bmk);
                st_f2(t + T_BMV * TS, bmv);
                st_f2(t + T_BRK * TS, brk);
                st_f2(t + T_BRV * TS, brv);
            }
        }
        __syncthreads();

        // ---- 2. four walks over the segments, one thread per channel each: forwards for k and
        // for v (Lam, P, F, Y entering each segment, and E), backwards for k and for v (D and the
        // mu, rho carries entering from the right)
        {
            const int w = tid / SW, ch = tid % SW;
            float *t = tab + ch;
            constexpr int GS = 8;                      // segments loaded per batch
            if (w < 2) {
                const int TK = w ? T_KNV : T_KNK, TF = w ? T_BFV : T_BFK, TY = w ? T_YPV : T_YPK;
                float pn = 1.f, l = 0.f, pp = 1.f, f = 0.f, y = 0.f;
#pragma unroll
                for (int u0 = 0; u0 < SEGS; u0 += GS) {
                    float an[GS], kn[GS], a[GS], bf[GS], yp[GS];
#pragma unroll
                    for (int u = 0; u < GS; ++u) {
                        an[u] = t[T_AN * TS + (u0 + u) * SW];
                        kn[u] = t[TK * TS + (u0 + u) * SW];
                        a[u] = t[T_A * TS + (u0 + u) * SW];
                        bf[u] = t[TF * TS + (u0 + u) * SW];
                        yp[u] = t[TY * TS + (u0 + u) * SW];
                    }
#pragma unroll
                    for (int u = 0; u < GS; ++u) {
                        float *x = t + (u0 + u) * SW;
                        if (w == 0) {
                            x[T_PN * TS] = pn;
                            x[T_P * TS] = pp;
                        }
                        x[TK * TS] = l;
                        x[TF * TS] = f;
                        x[TY * TS] = y;
                        y = fmaf(a[u], y, fmaf(bf[u], l, yp[u] * pn));
                        f = fmaf(a[u], f, bf[u]);
                        pp *= a[u];
                        l = fmaf(pn, kn[u], l);
                        pn *= an[u];
                    }
                }
                Etab[w * SW + ch] = f;
            } else {
                const int TM = w == 3 ? T_BMV : T_BMK, TR = w == 3 ? T_BRV : T_BRK;
                float dd = 1.f, m = 0.f, r = 0.f;
#pragma unroll
                for (int u0 = SEGS - GS; u0 >= 0; u0 -= GS) {
                    float a[GS], bm[GS], br[GS];
#pragma unroll
                    for (int u = 0; u < GS; ++u) {
                        a[u] = t[T_A * TS + (u0 + u) * SW];
                        bm[u] = t[TM * TS + (u0 + u) * SW];
                        br[u] = t[TR * TS + (u0 + u) * SW];
                    }
#pragma unroll
                    for (int u = GS - 1; u >= 0; --u) {
                        float *x = t + (u0 + u) * SW;
                        if (w == 2) x[T_D * TS] = dd;
                        x[TM * TS] = m;
                        x[TR * TS] = r;
                        m = fmaf(a[u], m, bm[u]);
                        r = fmaf(a[u], r, br[u]);
                        dd *= a[u];
                    }
                }
            }
        }
        __syncthreads();

        // ---- 3. my rows: gradients, and U of this block for the next one
        {
            f2_t xk[R][2], xv[R][2], ek[R][2], ev[R][2];
            load_xe(xk, xv, ek, ev);
            f2_t dk[R][2], dv[R][2], da[R][2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float *t = tab + seg * SW + (q ? HSW : 0) + 2 * cl;
                const f2_t pn = ld_f2(t + T_PN * TS);
                const f2_t lk0 = ld_f2(t + T_KNK * TS), lv0 = ld_f2(t + T_KNV * TS);
                const f2_t Ek = ld_f2(Etab + (q ? HSW : 0) + 2 * cl);
                const f2_t Ev = ld_f2(Etab + SW + (q ? HSW : 0) + 2 * cl);
                // forwards over my rows: Lam at each row; F, P, Y before each row; F at each row
                f2_t Lk[R], Lv[R], Fmk[R + 1], Fmv[R + 1], Pm[R], Ymk[R], Ymv[R];
                Fmk[0] = ld_f2(t + T_BFK * TS);
                Fmv[0] = ld_f2(t + T_BFV * TS);
                Pm[0] = ld_f2(t + T_P * TS);
                Ymk[0] = ld_f2(t + T_YPK * TS);
                Ymv[0] = ld_f2(t + T_YPV * TS);
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    const f2_t gi = g[i][q], og = gate_complement2(gi);
                    Lk[i] = f2_fma(pn, lk[i][q], lk0);
                    Lv[i] = f2_fma(pn, lv[i][q], lv0);
                    Fmk[i + 1] = f2_fma(gi, Fmk[i], f2_mul(og, xk[i][q]));
                    Fmv[i + 1] = f2_fma(gi, Fmv[i], f2_mul(og, xv[i][q]));
                    if (i + 1 < R) {
                        Pm[i + 1] = f2_mul(Pm[i], gi);
                        Ymk[i + 1] = f2_fma(gi, Ymk[i], f2_mul(f2_mul(og, xk[i][q]), Lk[i]));
                        Ymv[i + 1] = f2_fma(gi, Ymv[i], f2_mul(f2_mul(og, xv[i][q]), Lv[i]));
                    }
                }
                // backwards: D after each row, mu and rho from the carries entering from the right
                f2_t D = ld_f2(t + T_D * TS);
                f2_t mk = ld_f2(t + T_BMK * TS), mv = ld_f2(t + T_BMV * TS);
                f2_t rk = ld_f2(t + T_BRK * TS), rv = ld_f2(t + T_BRV * TS);
#pragma unroll
                for (int i = R - 1; i >= 0; --i) {
                    const f2_t gi = g[i][q], og = gate_complement2(gi);
                    const f2_t muk = f2_add(ek[i][q], mk), muv = f2_add(ev[i][q], mv);
                    const f2_t rok = f2_fma(ek[i][q], U1k[i][q], rk);
                    const f2_t rov = f2_fma(ev[i][q], U1v[i][q], rv);
                    // dx = (1 - g) (mu + D Lam)
                    dk[i][q] = f2_mul(og, f2_fma(D, Lk[i], muk));
                    dv[i][q] = f2_mul(og, f2_fma(D, Lv[i], muv));
                    // dg = mu (F(j-1) - x) + P(j-1) rho + D (Y(j-1) - x Lam), k and v summed
                    f2_t sg = f2_mul(muk, f2_fma(xk[i][q], kNeg2, Fmk[i]));
                    sg = f2_fma(muv, f2_fma(xv[i][q], kNeg2, Fmv[i]), sg);
                    sg = f2_fma(Pm[i], f2_add(rok, rov), sg);
                    sg = f2_fma(D, f2_add(f2_fma(f2_mul(xk[i][q], Lk[i]), kNeg2, Ymk[i]),
                                          f2_fma(f2_mul(xv[i][q], Lv[i]), kNeg2, Ymv[i])), sg);
                    da[i][q] = f2_mul(f2_mul(gi, og), sg);
                    // U of this block at row j + 1: E - D(j) F(j)
                    U1k[i][q] = f2_fma(f2_mul(D, kNeg2), Fmk[i + 1], Ek);
                    U1v[i][q] = f2_fma(f2_mul(D, kNeg2), Fmv[i + 1], Ev);
                    mk = f2_mul(gi, muk);
                    mv = f2_mul(gi, muv);
                    rk = f2_mul(gi, rok);
                    rv = f2_mul(gi, rov);
                    D = f2_mul(gi, D);
                }
            }
            if (!prep) {
                void *ok = c < 0 ? p.dpk : p.dk, *ov = c < 0 ? p.dpv : p.dv, *oa = c < 0 ? p.dpa : p.da;
#pragma unroll
                for (int i = 0; i < R; ++i) {
                    const int j = j0 + i;
                    if (j >= rows) continue;
                    const size_t grow = c < 0 ? (size_t)bh * LW + j : (size_t)bh * p.T + (size_t)c * LW + j;
                    const size_t o = grow * rowstride + col + (size_t)2 * cl * C::EB;
                    WbLane<E>::store(static_cast<uint8_t *>(ok) + o, static_cast<uint8_t *>(ok) + o + halfoff, dk[i]);
                    WbLane<E>::store(static_cast<uint8_t *>(ov) + o, static_cast<uint8_t *>(ov) + o + halfoff, dv[i]);
                    WbLane<E>::store(static_cast<uint8_t *>(oa) + o, static_cast<uint8_t *>(oa) + o + halfoff, da[i]);
                }
            }
        }
        u_bh = bh;
        u_c = c;
        __syncthreads();            // this item's stages and the tables are free
        const WbItem na = wb_next(ca, f0, f1, p.nblk, cmin, has_prev);
        const WbItem nk = wb_next(ck, f0, f1, p.nblk, cmin, has_prev);
        issue_agd(na, it_k % C::NAGD);
        issue_kv(nk, it_k & 1);
        cp_async_commit();
    }
    cp_async_wait_0();              // no copy may land after the CTA has left the SM
}

template <typename E>
static int launch_one(const WindowBwdParams &p, void *stream) {
    using C = WbCfg<E>;
    auto kern = window_bwd_kernel<E>;
    static std::atomic<uint64_t> attr_done{0};
    const int st = set_smem_attr(reinterpret_cast<const void *>(kern), C::SMEM, &attr_done);
    if (st != RAT_OK) return st;
    const int sms = current_sm_count();
    if (sms <= 0) return RAT_ERR_CUDA;
    // ns CTAs (one per slice) per range of (b, h, block) items, at most one CTA per SM
    const int ns = p.d / C::SW;
    const int cmin = p.dpk != nullptr ? -1 : 0;
    const long long total = (long long)p.BH * (p.nblk - cmin);
    long long nranges = sms / ns;
    if (nranges < 1) nranges = 1;
    if (nranges > total) nranges = total;
    const unsigned grid = (unsigned)(nranges * ns);
    kern<<<grid, C::THREADS, C::SMEM, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

int launch_window_bwd(const WindowBwdParams &p, int dtype, void *stream) {
    if (p.d != 64 && p.d != 128) return RAT_ERR_UNSUPPORTED;
    return dtype == RAT_F32 ? launch_one<float>(p, stream) : launch_one<__nv_bfloat16>(p, stream);
}

}  // namespace rat
