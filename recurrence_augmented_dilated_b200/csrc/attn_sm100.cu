// attn_sm100.cu -- bf16 causal dilated attention prefill on tcgen05 tensor cores (sm_100a).
//
// RAT+ abstract ("dilated attention ... optionally with local windows ... hybrid layer/head
// compositions"); "RAT+ Deep Dive" section 3.1 (attention FLOPs T/D) and section 6 (per-head
// dilation).  Query t of head h attends to
//     S(t) = { t-We < j <= t }  U  { j <= t-We : j mod D_h = D_h - 1 },   We = max(W, 1),
// i.e. its local window (itself included) and the chunk ends older than the window; a head
// with D_h = 1 is dense causal attention.
//
// One CTA computes one 128-query tile of one (b, h) with two key streams:
//   * the dilated stream -- the chunk ends i*D + D - 1, read through a TMA tensor map whose row
//     stride is D rows of the recurrence output, so the gather costs nothing but a descriptor;
//   * the window stream -- the contiguous band of positions the tile's windows cover.
// Both are cut into blocks of BN keys (64 by default, two CTAs per SM; 128 selectable, one CTA
// per SM).  Per block:
//   S = Q K^T   (tcgen05.mma, bf16 operands from 128B-swizzled smem, f32 accumulator in TMEM,
//                double-buffered so the next block's product overlaps this block's softmax);
//   softmax     (one thread per query row reads its S row from TMEM, masks it to S(t), keeps a
//                running max and sum; the max is only moved -- and O rescaled in TMEM -- when
//                it grows by more than 2^8, which keeps the result exact and rescales rare);
//   O += P V    (P written back as bf16 into the first columns of its S buffer in TMEM and read
//                from there as the A operand; V an MN-major smem operand).
// With W <= 1 the self key stays out of the blocks: its k~ and v~ rows are read directly and it
// joins the softmax and O in registers.  Attention sinks arrive as one more key block.  A
// template variant adds top-k chunk selection (see attn_sm100_kernel).
// Roles: warp 0 issues TMA loads (2-stage K and V rings with separate lifetimes), warp 1
// allocates TMEM and issues the MMAs, warps 2-5 do RoPE on Q (in smem), the softmax and the
// epilogue (O / l -> bf16 -> smem -> TMA store).  Every mbarrier wait is bounded; on expiry the
// CTA records RAT_ERR_TIMEOUT in a module error word, stops all roles, waits for its own async
// work and frees TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "tc.cuh"

namespace rat {

__device__ int g_attn_error;     // first device-side error of the attention kernel
__device__ unsigned g_attn_where; // where it happened: (site << 24) | (block << 8) | parity
__device__ unsigned g_attn_waiting; // bit s set: a wait at site s was in progress when a CTA aborted

// (cos, sin)(l * theta_f) for l < 16 and the 64 RoPE frequencies, [f][l], formed on the host in
// float64; the producer copies a launch's table next to Q.  kRelSlots tables per device, one per
// distinct frequency set (RoPE base), each written once and never replaced.
constexpr int kRelSlots = 16;
constexpr int kRelL = 16;
__device__ float2 g_rope_rel[kRelSlots][64 * kRelL];

namespace {

constexpr int BM = 128;               // query rows per tile
constexpr int DHEAD = 128;
constexpr int NS = 2;                 // K/V pipeline stages
constexpr int kThreads = 192;         // warp 0: TMA, warp 1: MMA, warps 2-5: softmax / epilogue
constexpr uint32_t QSUB = BM * 128;   // one [128 rows][64 bf16] 128B-swizzled sub-tile of Q / O
constexpr int kMaxDil = 4;
constexpr float kRescaleLog2 = 8.0f;             // move the running max only when it grows by > 2^8
constexpr uint32_t kRelBytes = 64 * kRelL * 8;    // the RoPE table g_rope_rel
constexpr int kBasStride = 65;                    // padded row of the per-tile base rotations

// Shared-memory / TMEM plan for key blocks of BN keys.
template <int BN>
struct Cfg {
    static constexpr uint32_t KSUB = BN * 128;          // [BN keys][64 bf16] sub-tile
    static constexpr uint32_t KTILE = 2 * KSUB;         // one K (or V) block: two d-halves
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + 2 * QSUB;
    static constexpr uint32_t OFF_V = OFF_K + NS * KTILE;
    // 96 KiB + barriers for 64-key blocks: two CTAs stay within the 196 KiB shared-memory
    // carveout, which leaves the rest of the SM's 256 KiB to L1
    static constexpr uint32_t OFF_BAR = OFF_V + NS * KTILE;
    static constexpr uint32_t SMEM_BYTES = OFF_BAR + 256;
    // top-k variant: a bitmap of the key blocks that hold some row's selected chunks
    static constexpr uint32_t OFF_MAP = OFF_BAR + 256;
    static constexpr uint32_t MAP_WORDS = 64;           // 2048 blocks: positions below 131072
    static constexpr uint32_t SMEM_TOPK = OFF_MAP + MAP_WORDS * 4;
    static constexpr uint32_t COL_S1 = BN;              // S buffers at columns 0 and BN; the bf16
                                                        // P of a block overwrites the first BN/2
                                                        // columns of its S buffer
    static constexpr uint32_t COL_O = 2 * BN;           // O: 128 columns after them
    static constexpr uint32_t TMEM_COLS = BN == 64 ? 256 : 512;
    static constexpr int MIN_CTAS = BN == 64 ? 2 : 1;   // CTAs resident per SM
};

struct Params {
    CUtensorMap tm_q;                              // (d, T, B*H) bf16, box (64, 128, 1), 128B swizzle
    CUtensorMap tm_k, tm_v;                        // same tensors, box (64, BN, 1)
    CUtensorMap tm_kd[kMaxDil], tm_vd[kMaxDil];    // chunk ends of one dilation: (d, T/D, B*H)
    CUtensorMap tm_o;                              // output (d, T, B*H), box (64, 32, 1), 128B swizzle
    const void *kg, *vg;                           // k~, v~ (the self key when W <= 1)
    void *og;                                      // output, written row by row
    int B, H, T, W, ntiles;
    long long pos0;
    int rope;
    float scale_log2;
    int head_of[kMaxHeads];   // heads sorted by dilation, smallest (most keys) first
    int Dh[kMaxHeads];
    int dslot[kMaxHeads];     // head -> index into tm_kd / tm_vd (-1 when D == 1)
    // work order: groups of heads with equal D, in head_of order; inside a group, tiles from
    // the last (most keys) to the first, all (b, head) of a tile row together
    int ngroups;
    int grp_item0[kMaxHeads + 1];   // first linear block index of each group
    int grp_head0[kMaxHeads];       // first index into head_of
    int grp_nheads[kMaxHeads];
    int rope_f32;             // positions small enough for float32 angles (pos0 + T <= 2^13)
    int n_sink;               // attention sinks (n_sink < D of every dilated head, <= BN)
    int top_k;                // top-k variant: chunks selected per row (1 .. 16)
    float *lse;               // [B*H][T] or null: log2 of each row's softmax denominator
    const float2 *rope_rel;   // device table [64 f][16 l] of (cos, sin)(l theta_f), see g_rope_rel
    float theta_f[64];
    double theta[64];
};

RAT_DEVICE int floordiv(int a, int b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

// Key blocks of one tile: ns sink blocks (0 or 1: positions 0 .. n_sink-1), nd dilated blocks
// (compressed indices BN*j ..), then nw window blocks starting at position ws (contiguous).
// Dense heads have ns = nd = 0 and ws = 0.  Sinks come here only when no chunk end is a sink
// (n_sink < D) and n_sink <= BN, so the three sets stay disjoint with contiguous columns.
struct Plan {
    int ns, nd, nw, ws, D, We, n_sink;
    bool dense;
    bool self_reg;    // We == 1 (dilated head): the self key is handled in registers, no window blocks
};
template <int BN>
RAT_DEVICE Plan make_plan(int t0, int D, int W, int T, int n_sink, bool regs_self = true) {
    Plan pl;
    pl.D = D;
    pl.We = W > 1 ? W : 1;
    pl.dense = D == 1;
    pl.self_reg = regs_self && !pl.dense && pl.We == 1;
    pl.n_sink = n_sink;
    const int tmax = t0 + BM - 1;
    // a sink block when some query of the tile has a sink older than its window
    pl.ns = (!pl.dense && n_sink > 0 && tmax - pl.We + 1 > 0) ? 1 : 0;
    if (pl.dense) {
        pl.nd = 0;
        pl.ws = 0;
        pl.nw = (tmax + 1 + BN - 1) / BN;
    } else {
        int ndk = tmax - pl.We + 1 >= D ? (tmax - pl.We + 1) / D : 0;  // chunk ends <= tmax - We
        const int cap = T / D;
        if (ndk > cap) ndk = cap;
        pl.nd = (ndk + BN - 1) / BN;
        pl.ws = t0 - pl.We + 1 > 0 ? t0 - pl.We + 1 : 0;
        pl.nw = pl.self_reg ? 0 : (tmax + 1 - pl.ws + BN - 1) / BN;
    }
    return pl;
}

// Columns [c_lo, c_hi] of block j that query t may attend to.
template <int BN>
RAT_DEVICE void block_range(const Plan &pl, int j, int t, int &c_lo, int &c_hi) {
    if (j < pl.ns) {
        // sinks older than the window: positions 0 .. min(n_sink, t - We + 1) - 1
        c_lo = 0;
        c_hi = min(pl.n_sink, t - pl.We + 1) - 1;
        return;
    }
    j -= pl.ns;
    if (j < pl.nd) {
        // chunk end i = BN j + c is attended iff i*D + D - 1 <= t - We
        c_lo = 0;
        c_hi = floordiv(t - pl.We - pl.D + 1, pl.D) - BN * j;
    } else {
        const int base = pl.ws + BN * (j - pl.nd);
        c_hi = t - base;
        c_lo = pl.dense ? -(1 << 30) : t - pl.We + 1 - base;
    }
}

struct Shared {
    // K and V of a stage have separate lifetimes: K is free once S has read it, V once PV has
    uint64_t q_full, q_ready, k_full[NS], v_full[NS], k_empty[NS], v_empty[NS];
    uint64_t s_full[2], p_full[2], o_ready[2], fin;
    uint64_t sel_free[2], sel_ready;   // top-k variant: selection scores read, selection published
    uint32_t tmem;
    volatile int abort;
};
static_assert(sizeof(Shared) <= 256, "barriers fit the 256 bytes reserved after the tiles");

// Bounded mbarrier wait that also gives up as soon as another role aborted; an expired wait
// records RAT_ERR_TIMEOUT and its site (see g_attn_where).
RAT_DEVICE bool wait_bar(Shared &sh, uint64_t *bar, uint32_t parity, uint32_t site = 0, uint32_t blk = 0) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (sh.abort) {
            atomicOr(&g_attn_waiting, 1u << site);
            return false;
        }
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            sh.abort = 1;
            if (atomicCAS(&g_attn_error, 0, RAT_ERR_TIMEOUT) == 0)
                g_attn_where = (site << 24) | ((blk & 0xffffu) << 8) | parity;
            return false;
        }
    }
}

// Bounded wait that ignores aborts: a role draining its own asynchronous copies before exit.
RAT_DEVICE void wait_drain(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
}

// cos/sin of pos * theta: angle in float64 reduced by 2*pi (two-term constant), then the
// special-function-unit sincos on [-pi, pi] (absolute error ~1e-6, far below bf16 rounding).
RAT_DEVICE void rope_cs_fast(long long pos, double theta, float &c, float &s) {
    const double kTwoPiHi = 6.283185307179586, kTwoPiLo = 2.4492935982947064e-16;
    const double ang = (double)pos * theta;
    const double n = rint(ang * 0.15915494309189535);
    double r = fma(-n, kTwoPiHi, ang);
    r = fma(-n, kTwoPiLo, r);
    __sincosf((float)r, &s, &c);
}

// Index of the n-th (0-based) set bit of a bitmap of `words` 32-bit words; -1 if there is none.
RAT_DEVICE int nth_set(const uint32_t *bm, int words, int n) {
    for (int w = 0; w < words; ++w) {
        uint32_t x = bm[w];
        const int c = __popc(x);
        if (n < c) {
            for (; n > 0; --n) x &= x - 1;
            return 32 * w + __ffs(x) - 1;
        }
        n -= c;
    }
    return -1;
}
RAT_DEVICE int count_set(const uint32_t *bm, int words) {
    int n = 0;
    for (int w = 0; w < words; ++w) n += __popc(bm[w]);
    return n;
}

// 16 bytes global -> shared without passing through registers (completion: cp_async_wait_all)
RAT_DEVICE void cp_async16(void *sdst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(smem_u32(sdst)), "l"(gsrc) : "memory");
}
RAT_DEVICE void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

RAT_DEVICE uint32_t swz(uint32_t row, uint32_t chunk) {   // 128B swizzle inside a sub-tile
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// SELF: the launch may have heads whose self key is kept in registers (W <= 1); launches with a
// window (W > 1) compile without that code.
// TOPK: top-k chunk selection combined with dilation ("RAT+ Deep Dive" section 4).  A selection
// phase first runs S over the chunk-end blocks alone; each row keeps its 16 best chunks (by
// chunk-end score, ties to the earlier chunk) in registers, and the 64-key blocks holding the
// positions of every row's top_k chunks are marked in a shared bitmap.  The main loop then
// visits, between the chunk-end and the window blocks, each marked block once, each row keeping
// the columns of its own selected chunks (their chunk ends are keys already).  The self key
// stays in the window blocks.
template <int BN, bool SELF, bool TOPK = false>
__global__ void __launch_bounds__(kThreads, Cfg<BN>::MIN_CTAS)
attn_sm100_kernel(const __grid_constant__ Params p) {
    using C = Cfg<BN>;
    extern __shared__ __align__(1024) uint8_t smem[];
    // the 128B-swizzled tiles need a 1024-byte aligned base; every thread sees the same address,
    // so this early exit is CTA-uniform and happens before any barrier, TMA or TMEM use
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(&g_attn_error, 0, RAT_ERR_UNSUPPORTED);
        return;
    }
    Shared &sh = *reinterpret_cast<Shared *>(smem + C::OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // linear block index -> (tile, b, h): longest work first (see Params)
    const int L = (int)blockIdx.x;
    int g = 0;
    while (g + 1 < p.ngroups && L >= p.grp_item0[g + 1]) ++g;
    const int local = L - p.grp_item0[g];
    const int per_row = p.B * p.grp_nheads[g];
    const int tile = p.ntiles - 1 - local / per_row;
    const int t0 = tile * BM;
    const int b = (local % per_row) / p.grp_nheads[g];
    const int h = p.head_of[p.grp_head0[g] + (local % per_row) % p.grp_nheads[g]];
    const int bh = b * p.H + h;
    const Plan pl = make_plan<BN>(t0, p.Dh[h], p.W, p.T, p.n_sink, !TOPK);
    const bool self_reg = SELF && pl.self_reg;      // pl.self_reg implies W <= 1, hence SELF
    const int nb = pl.ns + pl.nd + pl.nw;           // (+ the selected blocks, top-k variant)
    const int nsel = TOPK ? pl.nd : 0;              // blocks of the selection phase
    uint32_t *bmap = reinterpret_cast<uint32_t *>(smem + Cfg<BN>::OFF_MAP);

    if (threadIdx.x == 0) {
        mbar_init(&sh.q_full, 1);
        mbar_init(&sh.q_ready, 128);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.k_empty[s], 1);
            mbar_init(&sh.v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) mbar_init(&sh.s_full[s], 1);
        // P of even / odd blocks: the softmax may finish block j while the MMA has not yet
        // consumed block j-1, but never block j+2 (that needs S(j+2), issued after PV(j))
        mbar_init(&sh.p_full[0], 128);
        mbar_init(&sh.p_full[1], 128);
        mbar_init(&sh.o_ready[0], 1);     // PV of even blocks
        mbar_init(&sh.o_ready[1], 1);     // PV of odd blocks
        mbar_init(&sh.fin, 1);
        if (TOPK) {
            mbar_init(&sh.sel_free[0], 128);
            mbar_init(&sh.sel_free[1], 128);
            mbar_init(&sh.sel_ready, 128);
            for (uint32_t w = 0; w < C::MAP_WORDS; ++w) bmap[w] = 0u;
        }
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(&sh.tmem, C::TMEM_COLS);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sh.tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const CUtensorMap *mk = pl.dense ? &p.tm_k : &p.tm_kd[max(p.dslot[h], 0)];
            const CUtensorMap *mv = pl.dense ? &p.tm_v : &p.tm_vd[max(p.dslot[h], 0)];
            tc::prefetch_tmap(&p.tm_q);
            tc::prefetch_tmap(mk);
            tc::prefetch_tmap(&p.tm_k);
            mbar_arrive_expect_tx(&sh.q_full, 2 * QSUB + (p.rope ? kRelBytes : 0u));
            tc::tma_load_3d(smem + C::OFF_Q, &p.tm_q, 0, t0, bh, &sh.q_full);
            tc::tma_load_3d(smem + C::OFF_Q + QSUB, &p.tm_q, 64, t0, bh, &sh.q_full);
            // RoPE: the relative rotation table goes to the second K stage, unused until Q is rotated
            if (p.rope) bulk_g2s(smem + C::OFF_K + C::KTILE, p.rope_rel, kRelBytes, &sh.q_full);
            // K runs one block ahead of V: S(j) needs K(j) long before PV(j) needs V(j), and a K
            // stage frees up as soon as its S has completed
            // first key row of block j: the sinks at row 0, a dilated block in the compressed
            // view, a window block in the plain one
            // (top-k variant: the ntk selected blocks sit between the chunk-end and the window
            // blocks; they are known once the selection is published)
            int ntk = 0;
            auto row_of = [&](int j) {
                if (j < pl.ns) return 0;
                j -= pl.ns;
                if (j < pl.nd) return BN * j;
                j -= pl.nd;
                if (TOPK && j < ntk) return BN * nth_set(bmap, C::MAP_WORDS, j);
                return pl.ws + BN * (j - ntk);
            };
            auto dil_blk = [&](int j) { return j >= pl.ns && j - pl.ns < pl.nd; };
            // K loads are counted over both phases (g), V loads over the main loop only (j)
            int k_issued = 0, v_issued = 0;
            bool go = true;
            if constexpr (TOPK) {
                for (int g = 0; g < nsel; ++g) {          // selection phase: chunk-end K blocks
                    const int s = g % NS;
                    if (g >= NS && !wait_bar(sh, &sh.k_empty[s], ((g / NS) - 1) & 1, 1, g)) { go = false; break; }
                    if (g == 1 && p.rope && !wait_bar(sh, &sh.q_ready, 0, 10, g)) { go = false; break; }
                    uint8_t *ks = smem + C::OFF_K + s * C::KTILE;
                    mbar_arrive_expect_tx(&sh.k_full[s], C::KTILE);
                    tc::tma_load_3d(ks, mk, 0, BN * g, bh, &sh.k_full[s]);
                    tc::tma_load_3d(ks + C::KSUB, mk, 64, BN * g, bh, &sh.k_full[s]);
                    k_issued = g + 1;
                }
                if (go && !wait_bar(sh, &sh.sel_ready, 0, 13, 0)) go = false;
                if (go) ntk = count_set(bmap, C::MAP_WORDS);
            }
            const int nbt = nb + ntk;
            for (int j = 0; go && j <= nbt; ++j) {
                if (j < nbt) {
                    const int g = nsel + j, s = g % NS;
                    if (g >= NS && !wait_bar(sh, &sh.k_empty[s], ((g / NS) - 1) & 1, 1, j)) break;
                    // with RoPE, stage 1 holds the softmax warps' rotation tables until Q is rotated
                    if (g == 1 && p.rope && !wait_bar(sh, &sh.q_ready, 0, 10, j)) break;
                    const CUtensorMap *tk = dil_blk(j) ? mk : &p.tm_k;
                    uint8_t *ks = smem + C::OFF_K + s * C::KTILE;
                    const int row = row_of(j);
                    mbar_arrive_expect_tx(&sh.k_full[s], C::KTILE);
                    tc::tma_load_3d(ks, tk, 0, row, bh, &sh.k_full[s]);
                    tc::tma_load_3d(ks + C::KSUB, tk, 64, row, bh, &sh.k_full[s]);
                    k_issued = g + 1;
                }
                if (j >= 1) {
                    const int jv = j - 1, s = jv % NS;
                    if (jv >= NS && !wait_bar(sh, &sh.v_empty[s], ((jv / NS) - 1) & 1, 11, jv)) break;
                    const CUtensorMap *tv = dil_blk(jv) ? mv : &p.tm_v;
                    uint8_t *vs = smem + C::OFF_V + s * C::KTILE;
                    mbar_arrive_expect_tx(&sh.v_full[s], C::KTILE);
                    tc::tma_load_3d(vs, tv, 0, row_of(jv), bh, &sh.v_full[s]);
                    tc::tma_load_3d(vs + C::KSUB, tv, 64, row_of(jv), bh, &sh.v_full[s]);
                    v_issued = jv + 1;
                }
            }
            if (sh.abort) {
                // let this CTA's own loads land before its shared memory goes away
                for (int g = max(0, k_issued - NS); g < k_issued; ++g) wait_drain(&sh.k_full[g % NS], (g / NS) & 1);
                for (int j = max(0, v_issued - NS); j < v_issued; ++j) wait_drain(&sh.v_full[j % NS], (j / NS) & 1);
                wait_drain(&sh.q_full, 0);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_QK = tc::idesc_bf16(BM, BN, 0);      // K^T: K-major B
            constexpr uint32_t IDESC_PV = tc::idesc_bf16(BM, DHEAD, 1);   // V: MN-major B
            const uint32_t sq = smem_u32(smem + C::OFF_Q);
            // S(g) = Q K(g)^T into S buffer g & 1, from K stage g % NS
            auto issue_s = [&](int g) {
                const int s = g % NS, sb = g & 1;
                const uint32_t sk = smem_u32(smem + C::OFF_K + s * C::KTILE);
                for (int kk = 0; kk < DHEAD / 16; ++kk) {
                    // 16 channels of Q (A, K-major) and of K (B, K-major): d-half kk/4, +32 B per step
                    const uint32_t qoff = (kk >> 2) * QSUB + (kk & 3) * 32;
                    const uint32_t koff = (kk >> 2) * C::KSUB + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem + sb * C::COL_S1, tc::smem_desc_sw128(sq + qoff, 16, 1024),
                                    tc::smem_desc_sw128(sk + koff, 16, 1024), IDESC_QK, kk > 0);
                }
                tc::mma_commit(&sh.s_full[sb]);
                tc::mma_commit(&sh.k_empty[s]);
            };
            bool ok = wait_bar(sh, &sh.q_ready, 0, 2);
            tc::fence_after_sync();
            int ntk = 0;
            if constexpr (TOPK) {
                for (int g = 0; ok && g < nsel; ++g) {        // selection phase: S only
                    if (!wait_bar(sh, &sh.k_full[g % NS], (g / NS) & 1, 3, g)) { ok = false; break; }
                    // S buffer g & 1 is free once the softmax warps have read S(g-2)
                    if (g >= 2 && !wait_bar(sh, &sh.sel_free[g & 1], ((g - 2) >> 1) & 1, 14, g)) { ok = false; break; }
                    tc::fence_after_sync();
                    issue_s(g);
                }
                // every selection-phase S has been read once the selection is published
                if (ok) ok = wait_bar(sh, &sh.sel_ready, 0, 13);
                if (ok) ntk = count_set(bmap, C::MAP_WORDS);
            }
            const int nbt = nb + ntk;
            for (int j = 0; ok && j <= nbt; ++j) {
                if (j < nbt) {
                    const int g = nsel + j;
                    if (!wait_bar(sh, &sh.k_full[g % NS], (g / NS) & 1, 3, j)) break;
                    // S buffer g & 1 holds P(j-2) until PV(j-2) has read it: wait for that PV to
                    // complete (this thread issued it, so the barrier is at most one phase ahead)
                    if (j >= 2 && !wait_bar(sh, &sh.o_ready[(j - 2) & 1], ((j - 2) >> 1) & 1, 4, j)) break;
                    tc::fence_after_sync();
                    issue_s(g);
                }
                if (j >= 1) {
                    const int jp = j - 1, s = jp % NS;
                    if (!wait_bar(sh, &sh.p_full[jp & 1], (jp >> 1) & 1, 5, jp)) break;
                    if (!wait_bar(sh, &sh.v_full[s], (jp / NS) & 1, 12, jp)) break;
                    tc::fence_after_sync();
                    const uint32_t sv = smem_u32(smem + C::OFF_V + s * C::KTILE);
                    const uint32_t pcol = ((nsel + jp) & 1) * C::COL_S1;     // P of block jp, in TMEM
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        // A = P[:, 16kk .. 16kk+15]: 8 TMEM columns of packed bf16 pairs
                        // B = V[16kk .. 16kk+15, :]  (MN-major: the two 64-channel atoms KSUB apart,
                        // 8-key groups 1 KiB apart)
                        const uint32_t boff = kk * 16 * 128;
                        tc::mma_bf16_ts(tmem + C::COL_O, tmem + pcol + kk * 8,
                                        tc::smem_desc_sw128(sv + boff, C::KSUB, 1024), IDESC_PV,
                                        (jp > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&sh.o_ready[jp & 1]);
                    tc::mma_commit(&sh.v_empty[s]);
                }
            }
            // all MMAs issued by this thread complete before TMEM can be released
            tc::mma_commit(&sh.fin);
            const uint64_t t_0 = globaltimer_ns();
            while (!mbar_try_wait(&sh.fin, 0) && globaltimer_ns() - t_0 < kWaitLimitNs) {
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;           // query row in the tile == TMEM lane
        const int t = t0 + r;
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        uint8_t *sQ = smem + C::OFF_Q;
        // Rows of the self key / value are read coalesced: in step k lane l holds the 16-byte chunk
        // (l & 15) of row q4*32 + 2k + (l >> 4) of the tile, so one warp load covers two whole rows.
        const int xc = lane & 15, xr = q4 * 32 + (lane >> 4);
        auto load_rows = [&](const void *base, uint4 *dst) {
            const uint4 *src = reinterpret_cast<const uint4 *>(base) + (size_t)bh * p.T * (DHEAD / 8) + xc;
            if (t0 + BM <= p.T) {
#pragma unroll
                for (int k = 0; k < 16; ++k) dst[k] = __ldg(src + (size_t)(t0 + xr + 2 * k) * (DHEAD / 8));
            } else {               // ragged last tile: rows past T repeat row T-1 (never stored)
#pragma unroll
                for (int k = 0; k < 16; ++k) dst[k] = __ldg(src + (size_t)min(t0 + xr + 2 * k, p.T - 1) * (DHEAD / 8));
            }
        };
        uint4 xrow[16];
        if (self_reg) load_rows(p.kg, xrow);         // k~ of the tile's rows, in flight with Q
        // rotate-half RoPE of the Q tile at positions pos0 + t.  Rotation of row 16g + l is
        // rot(base_g) * rot(l): rot(l theta_f) for l < 16 arrives with Q (the launch's table, copied
        // into the still-unused second K stage); while Q is in flight each warp tabulates
        // rot((pos0 + t0 + 16g) theta_f) for its own two row groups g in the second V stage; once Q
        // has landed each thread rotates its own row.
        const float2 *rel = reinterpret_cast<const float2 *>(smem + C::OFF_K + C::KTILE);  // [64 f][16 l]
        float2 *bas = reinterpret_cast<float2 *>(smem + C::OFF_V + C::KTILE);              // [8 g][kBasStride]
        if (p.rope) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int e = lane + 32 * k, g = 2 * q4 + (e >> 6), f = e & 63;
                const long long pos = p.pos0 + t0 + 16 * g;
                float cs, sn;
                if (p.rope_f32) rope_cs_f32((int)pos, p.theta_f[f], cs, sn);
                else rope_cs_fast(pos, p.theta[f], cs, sn);
                bas[g * kBasStride + f] = make_float2(cs, sn);
            }
            __syncwarp();
        }
        // waits are made warp-uniform: tcgen05.ld/st below are warp-collective
        bool ok = __all_sync(0xffffffffu, wait_bar(sh, &sh.q_full, 0, 6));
        if (ok && p.rope) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 *p1 = reinterpret_cast<uint4 *>(sQ + swz(r, c));
                uint4 *p2 = reinterpret_cast<uint4 *>(sQ + QSUB + swz(r, c));
                uint4 u1 = *p1, u2 = *p2;
                uint32_t a1[4] = {u1.x, u1.y, u1.z, u1.w}, a2[4] = {u2.x, u2.y, u2.z, u2.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float cs[2], sn[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int f = c * 8 + 2 * i + u;
                        const float2 b = bas[(r >> 4) * kBasStride + f], rl = rel[f * kRelL + (r & 15)];
                        cs[u] = b.x * rl.x - b.y * rl.y;
                        sn[u] = b.y * rl.x + b.x * rl.y;
                    }
                    const float x1l = bf16_lo(a1[i]), x1h = bf16_hi(a1[i]);
                    const float x2l = bf16_lo(a2[i]), x2h = bf16_hi(a2[i]);
                    a1[i] = pack_bf16(x1l * cs[0] - x2l * sn[0], x1h * cs[1] - x2h * sn[1]);
                    a2[i] = pack_bf16(x2l * cs[0] + x1l * sn[0], x2h * cs[1] + x1h * sn[1]);
                }
                *p1 = make_uint4(a1[0], a1[1], a1[2], a1[3]);
                *p2 = make_uint4(a2[0], a2[1], a2[2], a2[3]);
            }
            tc::fence_proxy_async_smem();
        }
        mbar_arrive(&sh.q_ready);

        float m_run = -INFINITY, l_run = 0.f;
        float w_self = 0.f;        // weight of the self key when it is kept in registers
        if (ok && self_reg) {
            // s_self = q^_t . k~_t: partial dots over 8 channels per lane for the 16 row pairs,
            // reduced over the 16 lanes of each half-warp by a transposing butterfly (after it,
            // lane l of half h holds the whole dot of row 2 (l & 15) + h), then handed to the lane
            // that owns the row
            __syncwarp();          // this warp's rows of q^ are rotated
            float part[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint4 qq = *reinterpret_cast<const uint4 *>(sQ + (xc >> 3) * QSUB + swz(xr + 2 * k, xc & 7));
                const uint32_t ku[4] = {xrow[k].x, xrow[k].y, xrow[k].z, xrow[k].w};
                const uint32_t qu[4] = {qq.x, qq.y, qq.z, qq.w};
                float d = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    d = fmaf(bf16_lo(qu[i]), bf16_lo(ku[i]), d);
                    d = fmaf(bf16_hi(qu[i]), bf16_hi(ku[i]), d);
                }
                part[k] = d;
            }
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1) {
                const bool upper = (lane & o) != 0;   // keeps the upper half of its o*2 values
#pragma unroll
                for (int i = 0; i < o; ++i) {
                    const float keep = upper ? part[i + o] : part[i];
                    const float send = upper ? part[i] : part[i + o];
                    part[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
            const float dot = __shfl_sync(0xffffffffu, part[0], ((lane & 1) << 4) | (lane >> 1));
            m_run = dot * p.scale_log2;
            w_self = 1.f;
        }
        float sv[BN];
        // top-k variant: this row's selected chunks (indices, -1: none), best first
        int sel[TOPK ? 16 : 1];
        int ntk = 0;
        if constexpr (TOPK) {
            float best[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) { best[q] = -INFINITY; sel[q] = -1; }
            for (int g = 0; ok && g < nsel; ++g) {
                const int sb = g & 1;
                if (!__all_sync(0xffffffffu, wait_bar(sh, &sh.s_full[sb], (g >> 1) & 1, 15, g))) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll
                for (int c = 0; c < BN / 32; ++c)
                    tc::tmem_ld32(tl + sb * C::COL_S1 + 32 * c, reinterpret_cast<uint32_t *>(sv) + 32 * c);
                tc::tmem_wait_ld();
                tc::fence_before_sync();
                mbar_arrive(&sh.sel_free[sb]);
                // candidate chunk i = BN g + c: wholly older than the window (its end <= t - We);
                // kept sorted, best first; an equal score does not displace an earlier chunk
                int c_lo, c_hi;
                block_range<BN>(pl, pl.ns + g, t, c_lo, c_hi);
                if (t >= p.T) c_hi = -1;
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    float v = sv[c];
                    if (c > c_hi || !(v > best[15])) continue;
                    int id = BN * g + c;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        if (v > best[q]) {
                            const float tv = best[q];
                            const int ti = sel[q];
                            best[q] = v;
                            sel[q] = id;
                            v = tv;
                            id = ti;
                        }
                    }
                }
            }
            // the key blocks holding the positions (below each chunk end) of the row's top_k chunks
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                if (q >= p.top_k) sel[q] = -1;
                if (sel[q] >= 0) {
                    const int b0 = sel[q] * pl.D / BN, b1 = (sel[q] * pl.D + pl.D - 2) / BN;
                    for (int b = b0; b <= b1; ++b) atomicOr(&bmap[b >> 5], 1u << (b & 31));
                }
            }
            mbar_arrive(&sh.sel_ready);
            if (ok) ok = __all_sync(0xffffffffu, wait_bar(sh, &sh.sel_ready, 0, 13));
            if (ok) ntk = count_set(bmap, C::MAP_WORDS);
        }
        const int nbt = nb + ntk;
        const int ndil = pl.ns + pl.nd;          // blocks before the selected ones
        int jdone = 0;
        for (int j = 0; ok && j < nbt; ++j) {
            const int sb = (nsel + j) & 1;
            if (!__all_sync(0xffffffffu, wait_bar(sh, &sh.s_full[sb], ((nsel + j) >> 1) & 1, 7, j))) { ok = false; break; }
            tc::fence_after_sync();
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
                tc::tmem_ld32(tl + sb * C::COL_S1 + 32 * c, reinterpret_cast<uint32_t *>(sv) + 32 * c);
            tc::tmem_wait_ld();

            // row max of the raw scores (scale > 0 commutes with max), as an 8-way tree; keys
            // outside S(t) become -inf (only blocks that cut the key set need the mask)
            float m8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) m8[u] = -INFINITY;
            if (TOPK && j >= ndil && j < ndil + ntk) {
                // a selected block: the columns inside this row's selected chunks, ends excluded
                const int base = BN * nth_set(bmap, C::MAP_WORDS, j - ndil);
                unsigned long long keep = 0ull;
#pragma unroll
                for (int q = 0; q < (TOPK ? 16 : 1); ++q) {
                    if (sel[q] < 0) continue;
                    const int lo = max(sel[q] * pl.D, base), hi = min(sel[q] * pl.D + pl.D - 2, base + BN - 1);
                    if (lo <= hi) keep |= ((~0ull) >> (63 - (hi - lo))) << (lo - base);
                }
#pragma unroll
                for (int c = 0; c < BN; ++c) sv[c] = (keep >> c) & 1ull ? sv[c] : -INFINITY;
            } else {
                int c_lo, c_hi;
                block_range<BN>(pl, j >= ndil + ntk ? j - ntk : j, t, c_lo, c_hi);
                if (!(c_lo <= 0 && c_hi >= BN - 1)) {
#pragma unroll
                    for (int c = 0; c < BN; ++c) sv[c] = (c >= c_lo && c <= c_hi) ? sv[c] : -INFINITY;
                }
            }
#pragma unroll
            for (int c = 0; c < BN; c += 2) m8[(c >> 1) & 7] = fmax3(m8[(c >> 1) & 7], sv[c], sv[c + 1]);
            const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                                   fmaxf(m8[6], m8[7])) * p.scale_log2;
            const float m_new = fmaxf(m_run, mx);
            const bool resc = m_new > m_run + kRescaleLog2;
            float alpha = 1.f;
            if (resc) {
                alpha = ex2_approx(m_run - m_new);
                l_run *= alpha;
                w_self *= alpha;
                m_run = m_new;
            }
            const float neg_mu = m_run == -INFINITY ? 0.f : -m_run;
            // exponents and row sum on float pairs (columns 2i, 2i+1)
            const f2_t sc2 = f2(p.scale_log2, p.scale_log2), mu2 = f2(neg_mu, neg_mu);
            f2_t s4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) s4[u] = f2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < BN / 2; ++i) {
                const f2_t x = f2_fma(f2(sv[2 * i], sv[2 * i + 1]), sc2, mu2);
                const f2_t e = f2(ex2_approx(f2lo(x)), ex2_approx(f2hi(x)));    // -inf -> 0
                sv[2 * i] = f2lo(e);
                sv[2 * i + 1] = f2hi(e);
                s4[i & 3] = f2_add(s4[i & 3], e);
            }
            const f2_t s2 = f2_add(f2_add(s4[0], s4[1]), f2_add(s4[2], s4[3]));
            l_run += f2lo(s2) + f2hi(s2);
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
                // the running max moved: O must hold PV of every earlier block before rescaling.
                // PV(j-1) completes phase (j-1)/2 of o_ready[(j-1)&1].  PV(j-3) is done (S(j) was
                // issued after it) and PV(j+1) cannot start before this block's P, so that barrier is
                // at most one phase ahead of the one waited for: the parity wait is unambiguous.
                if (!__all_sync(0xffffffffu, wait_bar(sh, &sh.o_ready[(j - 1) & 1], ((j - 1) >> 1) & 1, 8, j))) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tc::tmem_ld32(tl + C::COL_O + 32 * c, o);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tc::tmem_st32(tl + C::COL_O + 32 * c, o);
                }
            }
            // P row -> packed bf16 pairs -> the first BN/2 columns of this block's S buffer
#pragma unroll
            for (int c = 0; c < BN / 64; ++c) {
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) pk[i] = pack_bf16(sv[64 * c + 2 * i], sv[64 * c + 2 * i + 1]);
                tc::tmem_st32(tl + sb * C::COL_S1 + 32 * c, pk);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            mbar_arrive(&sh.p_full[j & 1]);
            jdone = j + 1;
        }
        // ---- epilogue: (O + w_self v~_t) / l -> bf16 rows in the Q buffer -> TMA stores of this
        // warp's 32 rows.  Every S product, the only reader of Q, has completed once the last S
        // buffer was seen full, so the self values are copied straight into this warp's rows
        // (128B-swizzled, no registers) while the last PV runs.
        bool have_o = ok && jdone == nbt;
        if (have_o && self_reg) {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.vg) + (size_t)bh * p.T * (DHEAD / 8) + xc;
#pragma unroll
            for (int k = 0; k < 16; ++k)       // rows past T repeat row T-1 (never stored)
                cp_async16(sQ + (xc >> 3) * QSUB + swz(xr + 2 * k, xc & 7),
                           src + (size_t)min(t0 + xr + 2 * k, p.T - 1) * (DHEAD / 8));
        }
        if (have_o && nbt > 0)
            have_o = __all_sync(0xffffffffu, wait_bar(sh, &sh.o_ready[(nbt - 1) & 1], ((nbt - 1) >> 1) & 1, 9, nbt));
        if (self_reg) {
            cp_async_wait_all();
            __syncwarp();
        }
        if (have_o) {
            tc::fence_after_sync();
            const float inv = 1.0f / (l_run + w_self);
            // the row's softmax denominator, for the backward (m_run is in log2-scaled units)
            if (p.lse && t < p.T) p.lse[(size_t)bh * p.T + t] = m_run + log2f(l_run + w_self);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                if (nbt > 0) {
                    tc::tmem_ld32(tl + C::COL_O + 32 * c, o);
                    tc::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
#pragma unroll
                for (int k8 = 0; k8 < 4; ++k8) {
                    const int ch = 4 * c + k8;                  // 16-byte chunk of the row
                    uint4 *dst = reinterpret_cast<uint4 *>(sQ + (ch >> 3) * QSUB + swz(r, ch & 7));
                    float f[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(o[8 * k8 + i]);
                    if (self_reg) {     // O += w_self * v~_t
                        const uint4 vv = *dst;
                        const uint32_t vu[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            f[2 * i] = fmaf(w_self, bf16_lo(vu[i]), f[2 * i]);
                            f[2 * i + 1] = fmaf(w_self, bf16_hi(vu[i]), f[2 * i + 1]);
                        }
                    }
                    *dst = make_uint4(pack_bf16(f[0] * inv, f[1] * inv), pack_bf16(f[2] * inv, f[3] * inv),
                                      pack_bf16(f[4] * inv, f[5] * inv), pack_bf16(f[6] * inv, f[7] * inv));
                }
            }
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && !sh.abort) {   // rows past T are clipped by the tensor map
                tc::tma_store_3d(&p.tm_o, sQ + q4 * 32 * 128, 0, t0 + q4 * 32, bh);
                tc::tma_store_3d(&p.tm_o, sQ + QSUB + q4 * 32 * 128, 64, t0 + q4 * 32, bh);
                tc::tma_store_commit_and_wait();
            }
            __syncwarp();
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, C::TMEM_COLS);
}


// ------------------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    // looked up once (a function-local static is initialised once, also under concurrent calls)
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        return nullptr;
    }();
    return fn;
}

// (d, rows, BH) bf16 view: row r of slice z at base + (z * slice_stride + r * row_stride) bytes;
// box (64 channels, box_rows, 1), 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t BH, uint64_t row_stride,
              uint64_t slice_stride, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)DHEAD, rows, BH};
    cuuint64_t strides[2] = {row_stride, slice_stride};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Fill the kernel parameters for key blocks of BN keys; returns the number of work items (or a
// negative rat_status).
template <int BN>
int fill_params(Params &p, const AttnSm100Args &a) {
    std::memset(&p, 0, sizeof(p));
    const uint64_t BH = (uint64_t)a.B * a.H, T = (uint64_t)a.T;
    const uint64_t row = DHEAD * 2, slice = T * row;
    if (!make_map(&p.tm_q, a.q, T, BH, row, slice, BM) || !make_map(&p.tm_o, a.o, T, BH, row, slice, 32) ||
        !make_map(&p.tm_k, a.k, T, BH, row, slice, BN) || !make_map(&p.tm_v, a.v, T, BH, row, slice, BN))
        return RAT_ERR_CUDA;
    // one strided map pair per distinct dilation > 1
    int dvals[kMaxDil], nd = 0;
    for (int h = 0; h < a.H; ++h) {
        const int D = a.Dh[h];
        p.Dh[h] = D;
        p.dslot[h] = -1;
        if (D == 1) continue;
        int slot = -1;
        for (int i = 0; i < nd; ++i)
            if (dvals[i] == D) slot = i;
        if (slot < 0) {
            if (nd == kMaxDil) return RAT_ERR_UNSUPPORTED;
            slot = nd;
            dvals[nd++] = D;
            const uint64_t cap = T / (uint64_t)D;
            const uint64_t off = (uint64_t)(D - 1) * row;
            if (cap > 0) {
                if (!make_map(&p.tm_kd[slot], static_cast<const uint8_t *>(a.k) + off, cap, BH, (uint64_t)D * row, slice, BN) ||
                    !make_map(&p.tm_vd[slot], static_cast<const uint8_t *>(a.v) + off, cap, BH, (uint64_t)D * row, slice, BN))
                    return RAT_ERR_CUDA;
            } else {   // no chunk end inside the sequence: the dilated stream is empty
                p.tm_kd[slot] = p.tm_k;
                p.tm_vd[slot] = p.tm_v;
            }
        }
        p.dslot[h] = slot;
    }
    // heads with the smallest dilation (most keys) first
    int order[kMaxHeads];
    for (int h = 0; h < a.H; ++h) order[h] = h;
    for (int i = 1; i < a.H; ++i)
        for (int k = i; k > 0 && a.Dh[order[k]] < a.Dh[order[k - 1]]; --k) {
            const int tmp = order[k];
            order[k] = order[k - 1];
            order[k - 1] = tmp;
        }
    for (int h = 0; h < a.H; ++h) p.head_of[h] = order[h];
    p.B = a.B; p.H = a.H; p.T = a.T; p.W = a.W;
    p.ntiles = (a.T + BM - 1) / BM;
    p.kg = a.k;
    p.vg = a.v;
    p.og = a.o;
    p.ngroups = 0;
    int items = 0;
    for (int i = 0; i < a.H;) {
        int k = i;
        while (k < a.H && a.Dh[order[k]] == a.Dh[order[i]]) ++k;
        p.grp_item0[p.ngroups] = items;
        p.grp_head0[p.ngroups] = i;
        p.grp_nheads[p.ngroups] = k - i;
        items += p.ntiles * a.B * (k - i);
        ++p.ngroups;
        i = k;
    }
    p.grp_item0[p.ngroups] = items;
    p.pos0 = a.pos0;
    p.rope = a.rope;
    p.rope_f32 = a.pos0 + (long long)a.T <= 8192 ? 1 : 0;
    p.n_sink = a.n_sink;
    p.top_k = a.top_k;
    p.lse = a.lse;
    p.scale_log2 = a.scale_log2;
    for (int c = 0; c < 64; ++c) {
        p.theta[c] = a.theta[c];
        p.theta_f[c] = (float)a.theta[c];
    }

    return items;
}

template <int BN, bool SELF, bool TOPK = false>
int launch_tiles(const Params &p, int items, void *stream) {
    using C = Cfg<BN>;
    constexpr uint32_t smem = TOPK ? C::SMEM_TOPK : C::SMEM_BYTES;
    static std::atomic<uint64_t> attr_done{0};
    const int st = set_smem_attr(reinterpret_cast<const void *>(attn_sm100_kernel<BN, SELF, TOPK>), smem, &attr_done);
    if (st != RAT_OK) return st;
    attn_sm100_kernel<BN, SELF, TOPK><<<(unsigned)items, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

template <int BN>
int launch_bn(const AttnSm100Args &a, const float2 *rel, void *stream) {
    Params p;          // copied into the launch's parameter space
    const int items = fill_params<BN>(p, a);
    if (items < 0) return items;
    p.rope_rel = rel;
    if constexpr (BN == 64) {
        if (a.top_k > 0) return launch_tiles<BN, false, true>(p, items, stream);
    }
    return a.W <= 1 ? launch_tiles<BN, true>(p, items, stream) : launch_tiles<BN, false>(p, items, stream);
}


}  // namespace

int g_attn_block_keys = 0;   // 0: automatic; 64 or 128 forces the key-block width

// The device table of a launch's RoPE frequencies.  The first call with a new frequency set
// writes it into a free slot on a library stream and waits for that copy before the slot is
// published, so a launch on any stream only ever reads a finished table; slots are never
// overwritten (queued launches may read them at any time).  Beyond kRelSlots distinct sets the
// call is refused (RAT_ERR_UNSUPPORTED), and a first use while `stream` is being captured is
// refused too (the upload cannot be part of a graph).
static int rope_rel_table(const double *theta, void *stream, const float2 **out) {
    struct Slot { double theta[64]; bool valid; };
    static std::mutex mu;
    static Slot slots[64][kRelSlots];
    static float2 *base[64];
    static cudaStream_t upload[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RAT_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!base[dev] && cudaGetSymbolAddress(reinterpret_cast<void **>(&base[dev]), g_rope_rel) != cudaSuccess)
        return RAT_ERR_CUDA;
    int free_slot = -1;
    for (int i = 0; i < kRelSlots; ++i) {
        if (!slots[dev][i].valid) {
            if (free_slot < 0) free_slot = i;
            continue;
        }
        if (std::memcmp(slots[dev][i].theta, theta, sizeof(double) * 64) == 0) {
            *out = base[dev] + (size_t)i * 64 * kRelL;
            return RAT_OK;
        }
    }
    if (free_slot < 0) return RAT_ERR_UNSUPPORTED;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cs) != cudaSuccess) return RAT_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return RAT_ERR_UNSUPPORTED;
    if (!upload[dev] && cudaStreamCreateWithFlags(&upload[dev], cudaStreamNonBlocking) != cudaSuccess)
        return RAT_ERR_CUDA;
    static float2 tab[64 * kRelL];      // guarded by mu
    for (int f = 0; f < 64; ++f)
        for (int l = 0; l < kRelL; ++l) {
            const double ang = (double)l * theta[f];
            tab[f * kRelL + l] = make_float2((float)std::cos(ang), (float)std::sin(ang));
        }
    if (cudaMemcpyToSymbolAsync(g_rope_rel, tab, sizeof(tab), (size_t)free_slot * sizeof(tab),
                                cudaMemcpyHostToDevice, upload[dev]) != cudaSuccess ||
        cudaStreamSynchronize(upload[dev]) != cudaSuccess)
        return RAT_ERR_CUDA;
    std::memcpy(slots[dev][free_slot].theta, theta, sizeof(double) * 64);
    slots[dev][free_slot].valid = true;
    *out = base[dev] + (size_t)free_slot * 64 * kRelL;
    return RAT_OK;
}

int launch_attn_sm100(const AttnSm100Args &a, void *stream) {
    if (a.d != DHEAD) return RAT_ERR_UNSUPPORTED;
    const float2 *rel = nullptr;
    if (a.rope) {
        const int st = rope_rel_table(a.theta, stream, &rel);
        if (st != RAT_OK) return st;
    }
    // (the top-k variant runs on 64-key blocks)
    const int bn = a.top_k > 0 ? 64 : g_attn_block_keys ? g_attn_block_keys : 64;
    return bn == 64 ? launch_bn<64>(a, rel, stream) : launch_bn<128>(a, rel, stream);
}

int attn_error_word(void *stream, bool clear) {
    int v = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return RAT_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_attn_error, sizeof(int)) != cudaSuccess) return RAT_ERR_CUDA;
    if (v != 0 && clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_attn_error, &zero, sizeof(int)) != cudaSuccess) return RAT_ERR_CUDA;
    }
    return v;
}

unsigned attn_error_where() {
    unsigned w = 0;
    if (cudaMemcpyFromSymbol(&w, g_attn_where, sizeof(unsigned)) != cudaSuccess) return 0xffffffffu;
    return w;
}

unsigned attn_error_waiting() {
    unsigned w = 0;
    if (cudaMemcpyFromSymbol(&w, g_attn_waiting, sizeof(unsigned)) != cudaSuccess) return 0xffffffffu;
    return w;
}

}  // namespace rat
