// attn_bwd_sm100.cu -- backward of the causal dilated attention on tcgen05 tensor cores
// (sm_100a, bf16 operands, float32 accumulation in TMEM).
//
// The forward (RAT+ abstract; "RAT+ Deep Dive" sections 3.1 and 6) lets query t of head h attend
//   S(t) = { t-We < j <= t }  U  { j <= t-We : j mod D_h = D_h - 1 },   We = max(W, 1),
// with p_t = softmax_j(scale <q^_t, k~_j>) and o_t = sum_j p_tj v~_j.  Training mixes dense and
// dilated samples ("RAT+ Deep Dive" section 2.2), which needs its reverse-mode derivative:
//   dp_tj = <dO_t, v~_j>,   ds_tj = p_tj (dp_tj - Delta_t),   Delta_t = <dO_t, o_t>,
//   dq^_t = scale sum_j ds_tj k~_j,   dk~_j = scale sum_t ds_tj q^_t,   dv~_j = sum_t p_tj dO_t,
// and dq = RoPE^T(dq^).  p_tj = 2^(scale log2e <q^_t, k~_j> - lse_t) from the forward's
// log2-sum-exp, so no running maximum is kept.  Every contraction runs on the tensor cores:
//
//   dq kernel  (one CTA per 128-query tile, like the forward): per block of BN keys (the
//              chunk ends through the strided tensor map, then the window band, the whole
//              prefix for a dense head; BN = 32 when every head is dilated, so that two CTAs
//              share an SM, else 64)
//                S = Q^ K^T and dP = dO V^T   (SS MMAs, 128 x BN each, into TMEM),
//                dS = P o (dP - Delta)        (softmax warps, one TMEM lane = query row each;
//                                              written back into TMEM as bf16),
//                dQ += dS K                   (TS MMA: dS from TMEM, K as the MN-major operand);
//              epilogue: dq = RoPE^T(scale dQ) -> bf16 rows.
//   dkv kernel (one CTA per block of 128 keys, the MMA's M): a chunk end (every key of a dense
//              head) is held by every query t >= its position, any other key by its window
//              queries t in [j, j + We - 1] only; so a block of chunk ends walks the 64-query
//              tiles from its first key to the end, a block of 128 consecutive positions (the
//              other keys, chunk ends masked out) walks the tiles of its window band.  Per tile
//                S^T = K Q^^T and dP^T = V dO^T   (SS MMAs, 128 x 64),
//                P^T, dS^T                        (softmax warps, one TMEM lane = key each),
//                dV += P^T dO,  dK += dS^T Q^     (TS MMAs, both operands' tiles reused);
//              epilogue: dk = scale dK, dv -> bf16 rows of the block's keys.
// q^ = RoPE(q) (bf16, as the forward's operand) and Delta come from the CUDA-core prep kernel.
// When the window is the self key alone (W <= 1), the key blocks of consecutive positions would
// hold one attending query per key: a dilated head's dq tiles then take the self term per row
// in their epilogue, and a CUDA-core kernel writes dk~, dv~ of the keys that are not chunk ends.
// Roles per CTA (192 threads): warp 0 issues TMA loads, warp 1 allocates TMEM and issues the
// MMAs (one elected thread), warps 2-5 do the elementwise work and the epilogue.  Every wait is
// bounded: an expired one records RAT_ERR_TIMEOUT in the workspace header, and the CTA stops
// its roles, waits for its own copies and MMAs, and frees TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "tc.cuh"

namespace rat {
namespace {

constexpr int DHEAD = 128;
constexpr int kThreads = 192;
constexpr int kMaxDil = 4;
constexpr uint32_t SUB128 = 128 * 128;   // [128 rows][64 bf16] 128B-swizzled sub-tile
constexpr uint32_t SUB64 = 64 * 128;     // [64 rows][64 bf16]

// ---- dq kernel: 128 queries x blocks of BN keys.  BN = 64: S[2], dP[2] and dQ take 384 TMEM
// columns (512 allocated), one CTA per SM; BN = 32: 256 columns and 96 KiB of shared memory,
// two CTAs per SM, for launches whose tiles are short (every head dilated).
template <int BN_>
struct DqCfg {
    static constexpr int BM = 128, BN = BN_;
    static constexpr uint32_t SUBK = BN * 128;           // [BN rows][64 bf16] 128B-swizzled sub-tile
    static constexpr uint32_t OFF_Q = 0;                 // q^ tile, two d-halves
    static constexpr uint32_t OFF_G = OFF_Q + 2 * SUB128;   // dO tile
    static constexpr uint32_t OFF_K = OFF_G + 2 * SUB128;   // two stages of a K block (two d-halves each)
    static constexpr uint32_t OFF_V = OFF_K + 2 * 2 * SUBK;
    static constexpr uint32_t OFF_BAR = OFF_V + 2 * 2 * SUBK;
    static constexpr uint32_t SMEM = OFF_BAR + 256;
    static constexpr uint32_t COL_S = 0, COL_P = 2 * BN, COL_Q = 4 * BN;   // S[2], dP[2], dQ
    static constexpr uint32_t TMEM_COLS = BN == 64 ? 512 : 256;
    static constexpr int MIN_CTAS = BN == 64 ? 1 : 2;
    static_assert(BN == 32 || BN == 64, "key blocks of 32 or 64");
};
namespace dqk {
constexpr int BM = 128;
}  // namespace dqk

// ---- dkv kernel: 128 keys x tiles of 64 queries
namespace dkv {
constexpr int BM = 128, BN = 64;
constexpr uint32_t OFF_K = 0;                       // key block, two d-halves
constexpr uint32_t OFF_V = OFF_K + 2 * SUB128;
constexpr uint32_t OFF_Q = OFF_V + 2 * SUB128;      // two stages of a q^ tile
constexpr uint32_t OFF_G = OFF_Q + 2 * 2 * SUB64;   // two stages of a dO tile
constexpr uint32_t OFF_BAR = OFF_G + 2 * 2 * SUB64;
constexpr uint32_t SMEM = OFF_BAR + 256;
constexpr uint32_t COL_S = 0, COL_P = 2 * BN, COL_V = 4 * BN, COL_K = 4 * BN + DHEAD;
}  // namespace dkv

struct Params {
    CUtensorMap tm_qh128, tm_g128;                 // q^, dO: (d, T, B*H), box (64, 128, 1)
    CUtensorMap tm_qh64, tm_g64;                   // box (64, 64, 1)
    CUtensorMap tm_kq, tm_vq, tm_k128, tm_v128;    // k~, v~ rows, boxes of the dq launch's BN / 128 rows
    CUtensorMap tm_kdq[kMaxDil], tm_vdq[kMaxDil];       // chunk ends of one dilation: (d, T/D, B*H)
    CUtensorMap tm_kd128[kMaxDil], tm_vd128[kMaxDil];
    const float *lse, *delta;                      // [B*H][T]
    const void *kg, *vg;                           // k~, v~ rows (self terms with W <= 1)
    void *dq, *dk, *dv;                            // outputs (B, H, T, d) bf16
    WsHeader *hdr;
    int B, H, T, W, ntiles;
    long long pos0;
    int rope;
    float scale, scale_log2;
    int Dh[kMaxHeads];
    int dslot[kMaxHeads];      // head -> strided map slot (-1 when D == 1)
    int head_of[kMaxHeads];    // heads sorted by dilation, smallest first
    // dq kernel work: groups of heads with equal D; inside a group tiles from the last (most
    // keys) to the first, all (b, head) of a tile row together
    int ngroups;
    int grp_item0[kMaxHeads + 1];
    int grp_head0[kMaxHeads];
    int grp_nheads[kMaxHeads];
    // dkv kernel work: sections (a) blocks of chunk ends of each group, then (b) blocks of
    // consecutive positions of each group with D > 1; inside a section block-major
    int nsec;
    int sec_item0[2 * kMaxDil + 3];
    int sec_grp[2 * kMaxDil + 2];
    int sec_type[2 * kMaxDil + 2];   // 0: chunk ends, 1: consecutive positions
    int sec_nblk[2 * kMaxDil + 2];
    double theta[64];
};

RAT_DEVICE int floordiv(int a, int b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

// Bounded mbarrier wait that also gives up as soon as another role aborted; an expired wait
// records RAT_ERR_TIMEOUT (detail: the wait site) in the workspace header.
RAT_DEVICE bool wait_bar(volatile int *abort, WsHeader *hdr, uint64_t *bar, uint32_t parity, uint32_t site) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            record_error(hdr, RAT_ERR_TIMEOUT, 0x400u | site);
            return false;
        }
    }
}
RAT_DEVICE void wait_drain(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < kWaitLimitNs) {
    }
}

// cos/sin of pos * theta: angle in float64 reduced by 2*pi (two-term constant), then the
// special-function-unit sincos on [-pi, pi] (absolute error ~1e-6, far below bf16 rounding).
RAT_DEVICE void rope_cs_sfu(long long pos, double theta, float &c, float &s) {
    const double kTwoPiHi = 6.283185307179586, kTwoPiLo = 2.4492935982947064e-16;
    const double ang = (double)pos * theta;
    const double n = rint(ang * 0.15915494309189535);
    double r = fma(-n, kTwoPiHi, ang);
    r = fma(-n, kTwoPiLo, r);
    __sincosf((float)r, &s, &c);
}

// Store 32 float values (channels c0 .. c0+31 of a row) as bf16: 64 bytes.
RAT_DEVICE void store_row32(uint8_t *row, int c0, const float *x) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        st_global_v4(row + (c0 + 8 * i) * 2, pack_bf16(x[8 * i], x[8 * i + 1]), pack_bf16(x[8 * i + 2], x[8 * i + 3]),
                     pack_bf16(x[8 * i + 4], x[8 * i + 5]), pack_bf16(x[8 * i + 6], x[8 * i + 7]));
}

struct BarsQ {
    uint64_t qd_full, kv_full[2], kv_empty[2], sdp_full[2], ds_full[2], dq_done[2], fin;
    uint32_t tmem;
    volatile int abort;
};
static_assert(sizeof(BarsQ) <= 256, "barriers fit the reserved bytes");

// ------------------------------------------------------------------------------ dq kernel
template <int BN_>
__global__ void __launch_bounds__(kThreads, DqCfg<BN_>::MIN_CTAS) attn_bwd_dq_sm100_kernel(const __grid_constant__ Params p) {
    using C = DqCfg<BN_>;
    constexpr int BM = C::BM, BN = C::BN;
    constexpr uint32_t SUBK = C::SUBK, OFF_Q = C::OFF_Q, OFF_G = C::OFF_G, OFF_K = C::OFF_K,
                       OFF_V = C::OFF_V, OFF_BAR = C::OFF_BAR, COL_S = C::COL_S, COL_P = C::COL_P,
                       COL_Q = C::COL_Q;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {     // CTA-uniform, before any barrier, TMA or TMEM use
        if (threadIdx.x == 0) record_error(p.hdr, RAT_ERR_UNSUPPORTED, 0x4ffu);
        return;
    }
    BarsQ &sh = *reinterpret_cast<BarsQ *>(smem + OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // linear block index -> (tile, b, h): longest work first
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
    const int D = p.Dh[h];
    const bool dense = D == 1;
    const int We = p.W > 1 ? p.W : 1;
    // key blocks: nd of chunk ends (compressed indices BN*j ..), then nw window blocks from ws
    const int tmax = t0 + BM - 1;
    // a dilated head whose window is the self key alone (W <= 1) takes the diagonal term per row
    // in the epilogue instead of two window blocks that would each hold one key per row
    const bool self_row = !dense && We == 1;
    int nd = 0, ws = 0, nw;
    if (dense) {
        nw = (min(tmax, p.T - 1) + 1 + BN - 1) / BN;
    } else {
        int ndk = tmax - We + 1 >= D ? (tmax - We + 1) / D : 0;
        ndk = min(ndk, p.T / D);
        nd = (ndk + BN - 1) / BN;
        ws = max(0, t0 - We + 1);
        nw = self_row ? 0 : (min(tmax, p.T - 1) + 1 - ws + BN - 1) / BN;
    }
    const int nb = nd + nw;

    if (threadIdx.x == 0) {
        mbar_init(&sh.qd_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.kv_full[s], 1);
            mbar_init(&sh.kv_empty[s], 1);
            mbar_init(&sh.sdp_full[s], 1);
            mbar_init(&sh.ds_full[s], 128);
            mbar_init(&sh.dq_done[s], 1);
        }
        mbar_init(&sh.fin, 1);
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
            const CUtensorMap *mk = dense ? &p.tm_kq : &p.tm_kdq[max(p.dslot[h], 0)];
            const CUtensorMap *mv = dense ? &p.tm_vq : &p.tm_vdq[max(p.dslot[h], 0)];
            tc::prefetch_tmap(&p.tm_qh128);
            tc::prefetch_tmap(&p.tm_g128);
            mbar_arrive_expect_tx(&sh.qd_full, 4 * SUB128);
            tc::tma_load_3d(smem + OFF_Q, &p.tm_qh128, 0, t0, bh, &sh.qd_full);
            tc::tma_load_3d(smem + OFF_Q + SUB128, &p.tm_qh128, 64, t0, bh, &sh.qd_full);
            tc::tma_load_3d(smem + OFF_G, &p.tm_g128, 0, t0, bh, &sh.qd_full);
            tc::tma_load_3d(smem + OFF_G + SUB128, &p.tm_g128, 64, t0, bh, &sh.qd_full);
            int issued = 0;
            for (int j = 0; j < nb; ++j) {
                const int s = j & 1;
                if (j >= 2 && !wait_bar(&sh.abort, p.hdr, &sh.kv_empty[s], ((j >> 1) - 1) & 1, 1)) break;
                const bool dil = j < nd;
                const CUtensorMap *tk = dil ? mk : &p.tm_kq, *tv = dil ? mv : &p.tm_vq;
                const int row = dil ? BN * j : ws + BN * (j - nd);
                uint8_t *ks = smem + OFF_K + s * 2 * SUBK, *vs = smem + OFF_V + s * 2 * SUBK;
                mbar_arrive_expect_tx(&sh.kv_full[s], 4 * SUBK);
                tc::tma_load_3d(ks, tk, 0, row, bh, &sh.kv_full[s]);
                tc::tma_load_3d(ks + SUBK, tk, 64, row, bh, &sh.kv_full[s]);
                tc::tma_load_3d(vs, tv, 0, row, bh, &sh.kv_full[s]);
                tc::tma_load_3d(vs + SUBK, tv, 64, row, bh, &sh.kv_full[s]);
                issued = j + 1;
            }
            if (sh.abort) {       // let this CTA's own loads land before its shared memory goes away
                for (int j = max(0, issued - 2); j < issued; ++j) wait_drain(&sh.kv_full[j & 1], (j >> 1) & 1);
                wait_drain(&sh.qd_full, 0);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = tc::idesc_bf16(BM, BN, 0);       // K^T, V^T: K-major B
            constexpr uint32_t IDESC_Q = tc::idesc_bf16(BM, DHEAD, 1);    // K: MN-major B
            const uint32_t sq = smem_u32(smem + OFF_Q), sg = smem_u32(smem + OFF_G);
            bool ok = wait_bar(&sh.abort, p.hdr, &sh.qd_full, 0, 2);
            tc::fence_after_sync();
            for (int j = 0; ok && j <= nb; ++j) {
                if (j < nb) {
                    const int s = j & 1;
                    if (!wait_bar(&sh.abort, p.hdr, &sh.kv_full[s], (j >> 1) & 1, 3)) break;
                    // buffers s hold dS(j-2) until its dQ MMA has read it
                    if (j >= 2 && !wait_bar(&sh.abort, p.hdr, &sh.dq_done[s], ((j - 2) >> 1) & 1, 4)) break;
                    tc::fence_after_sync();
                    const uint32_t sk = smem_u32(smem + OFF_K + s * 2 * SUBK);
                    const uint32_t sv = smem_u32(smem + OFF_V + s * 2 * SUBK);
                    for (int kk = 0; kk < DHEAD / 16; ++kk) {
                        const uint32_t ao = (kk >> 2) * SUB128 + (kk & 3) * 32;
                        const uint32_t bo = (kk >> 2) * SUBK + (kk & 3) * 32;
                        tc::mma_bf16_ss(tmem + COL_S + s * BN, tc::smem_desc_sw128(sq + ao, 16, 1024),
                                        tc::smem_desc_sw128(sk + bo, 16, 1024), IDESC_S, kk > 0);
                        tc::mma_bf16_ss(tmem + COL_P + s * BN, tc::smem_desc_sw128(sg + ao, 16, 1024),
                                        tc::smem_desc_sw128(sv + bo, 16, 1024), IDESC_S, kk > 0);
                    }
                    tc::mma_commit(&sh.sdp_full[s]);
                }
                if (j >= 1) {
                    const int jp = j - 1, s = jp & 1;
                    if (!wait_bar(&sh.abort, p.hdr, &sh.ds_full[s], (jp >> 1) & 1, 5)) break;
                    tc::fence_after_sync();
                    const uint32_t sk = smem_u32(smem + OFF_K + s * 2 * SUBK);
                    for (int kk = 0; kk < BN / 16; ++kk)
                        // A = dS[:, 16kk ..]: 8 TMEM columns of packed bf16 pairs; B = K[16kk .., :]
                        tc::mma_bf16_ts(tmem + COL_Q, tmem + COL_S + s * BN + kk * 8,
                                        tc::smem_desc_sw128(sk + kk * 16 * 128, SUBK, 1024), IDESC_Q,
                                        (jp > 0 || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&sh.dq_done[s]);
                    tc::mma_commit(&sh.kv_empty[s]);
                }
            }
            tc::mma_commit(&sh.fin);
            wait_drain(&sh.fin, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ dS rows + epilogue
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;           // query row in the tile == TMEM lane
        const int t = t0 + r;
        const bool live = t < p.T;
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        const float lse = live ? p.lse[(size_t)bh * p.T + t] : 0.f;
        const float dl = live ? p.delta[(size_t)bh * p.T + t] : 0.f;
        bool ok = true;
        for (int j = 0; j < nb; ++j) {
            const int s = j & 1;
            if (!__all_sync(0xffffffffu, wait_bar(&sh.abort, p.hdr, &sh.sdp_full[s], (j >> 1) & 1, 6))) { ok = false; break; }
            tc::fence_after_sync();
            float sv[BN], pv[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                tc::tmem_ld32(tl + COL_S + s * BN + 32 * c, reinterpret_cast<uint32_t *>(sv) + 32 * c);
                tc::tmem_ld32(tl + COL_P + s * BN + 32 * c, reinterpret_cast<uint32_t *>(pv) + 32 * c);
            }
            tc::tmem_wait_ld();
            // columns of block j this row attends to
            int c_lo, c_hi;
            if (j < nd) {
                c_lo = 0;
                c_hi = floordiv(t - We - D + 1, D) - BN * j;
            } else {
                const int base = ws + BN * (j - nd);
                c_hi = t - base;
                c_lo = dense ? 0 : t - We + 1 - base;
            }
            if (!live) c_hi = -1;
            uint32_t pk[BN / 2];
#pragma unroll
            for (int i = 0; i < BN / 2; ++i) {
                float d2[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c = 2 * i + u;
                    const float pr = (c >= c_lo && c <= c_hi) ? ex2_approx(fmaf(sv[c], p.scale_log2, -lse)) : 0.f;
                    d2[u] = pr * (pv[c] - dl);
                }
                pk[i] = pack_bf16(d2[0], d2[1]);
            }
            if constexpr (BN == 64) tc::tmem_st32(tl + COL_S + s * BN, pk);
            else tc::tmem_st16(tl + COL_S + s * BN, pk);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            mbar_arrive(&sh.ds_full[s]);
        }
        // the self term: dS_tt k~_t with p_tt = 2^(scale log2e <q^_t, k~_t> - lse_t) and
        // dp_tt = <dO_t, v~_t>; q^_t and dO_t come from this tile's rows in shared memory
        float ds_self = 0.f;
        uint4 ks[16];
        if (self_row && ok) {
            const size_t ro = ((size_t)bh * p.T + (live ? t : 0)) * DHEAD * 2;
            uint4 vs[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                ks[c] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.kg) + ro) + c);
                vs[c] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.vg) + ro) + c);
            }
            ok = __all_sync(0xffffffffu, wait_bar(&sh.abort, p.hdr, &sh.qd_full, 0, 8));
            float sd = 0.f, pd = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {       // 16-byte chunk c: channels 8c .. 8c+7
                const uint32_t off = (c >> 3) * SUB128 + r * 128u + ((((uint32_t)c & 7u) ^ ((uint32_t)r & 7u)) << 4);
                const uint4 qq = *reinterpret_cast<const uint4 *>(smem + OFF_Q + off);
                const uint4 gg = *reinterpret_cast<const uint4 *>(smem + OFF_G + off);
                const uint32_t qu[4] = {qq.x, qq.y, qq.z, qq.w}, gu[4] = {gg.x, gg.y, gg.z, gg.w};
                const uint32_t ku[4] = {ks[c].x, ks[c].y, ks[c].z, ks[c].w};
                const uint32_t vu[4] = {vs[c].x, vs[c].y, vs[c].z, vs[c].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    sd = fmaf(bf16_lo(qu[i]), bf16_lo(ku[i]), sd);
                    sd = fmaf(bf16_hi(qu[i]), bf16_hi(ku[i]), sd);
                    pd = fmaf(bf16_lo(gu[i]), bf16_lo(vu[i]), pd);
                    pd = fmaf(bf16_hi(gu[i]), bf16_hi(vu[i]), pd);
                }
            }
            const float pr = live ? ex2_approx(fmaf(sd, p.scale_log2, -lse)) : 0.f;
            ds_self = pr * (pd - dl);
        }
        if (ok && nb > 0)
            ok = __all_sync(0xffffffffu, wait_bar(&sh.abort, p.hdr, &sh.dq_done[(nb - 1) & 1], ((nb - 1) >> 1) & 1, 7));
        if (ok) {
            tc::fence_after_sync();
            uint8_t *row = static_cast<uint8_t *>(p.dq) + ((size_t)bh * p.T + t) * DHEAD * 2;
#pragma unroll
            for (int c = 0; c < 2; ++c) {        // channels [32c, 32c+32) and their partners + 64
                float lo[32], hi[32];
                if (nb > 0) {
                    tc::tmem_ld32(tl + COL_Q + 32 * c, reinterpret_cast<uint32_t *>(lo));
                    tc::tmem_ld32(tl + COL_Q + 64 + 32 * c, reinterpret_cast<uint32_t *>(hi));
                    tc::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) lo[i] = hi[i] = 0.f;
                }
                if (self_row) {                      // + dS_tt k~_t on channels 32c+i and 64+32c+i
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const uint4 kl = ks[(32 * c + i) >> 3], kh = ks[(64 + 32 * c + i) >> 3];
                        const uint32_t wl = ((i & 7) >> 1) == 0 ? kl.x : ((i & 7) >> 1) == 1 ? kl.y : ((i & 7) >> 1) == 2 ? kl.z : kl.w;
                        const uint32_t wh = ((i & 7) >> 1) == 0 ? kh.x : ((i & 7) >> 1) == 1 ? kh.y : ((i & 7) >> 1) == 2 ? kh.z : kh.w;
                        lo[i] = fmaf(ds_self, bf16_lo(wl), lo[i]);
                        lo[i + 1] = fmaf(ds_self, bf16_hi(wl), lo[i + 1]);
                        hi[i] = fmaf(ds_self, bf16_lo(wh), hi[i]);
                        hi[i + 1] = fmaf(ds_self, bf16_hi(wh), hi[i + 1]);
                    }
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float x = lo[i] * p.scale, y = hi[i] * p.scale;
                    if (p.rope) {     // RoPE^T: rotation by -(pos0 + t) theta_f
                        float cs, sn;
                        rope_cs_sfu(p.pos0 + t, p.theta[32 * c + i], cs, sn);
                        const float nx = fmaf(x, cs, y * sn), ny = fmaf(y, cs, -x * sn);
                        x = nx;
                        y = ny;
                    }
                    lo[i] = x;
                    hi[i] = y;
                }
                if (live) {
                    store_row32(row, 32 * c, lo);
                    store_row32(row, 64 + 32 * c, hi);
                }
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, C::TMEM_COLS);
}

struct BarsK {
    uint64_t kv_full, qd_full[2], qd_empty[2], sdp_full[2], pds_full[2], kv_done[2], fin;
    uint32_t tmem;
    volatile int abort;
};
static_assert(sizeof(BarsK) <= 256, "barriers fit the reserved bytes");

// Work item -> key block of one (b, h): type 0 = chunk ends [128 m, 128 m + 128) (every
// position for a dense head), type 1 = consecutive positions [128 m, 128 m + 128).
struct KBlock { int type, m, b, h; };
RAT_DEVICE KBlock kblock_of(const Params &p, int L) {
    int s = 0;
    while (s + 1 < p.nsec && L >= p.sec_item0[s + 1]) ++s;
    const int local = L - p.sec_item0[s];
    const int g = p.sec_grp[s];
    const int per = p.B * p.grp_nheads[g];
    KBlock kb;
    kb.type = p.sec_type[s];
    kb.m = local / per;
    kb.b = (local % per) / p.grp_nheads[g];
    kb.h = p.head_of[p.grp_head0[g] + (local % per) % p.grp_nheads[g]];
    return kb;
}

// ------------------------------------------------------------------------------ dkv kernel
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_dkv_sm100_kernel(const __grid_constant__ Params p) {
    using namespace dkv;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) record_error(p.hdr, RAT_ERR_UNSUPPORTED, 0x4feu);
        return;
    }
    BarsK &sh = *reinterpret_cast<BarsK *>(smem + OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const KBlock kb = kblock_of(p, (int)blockIdx.x);
    const int h = kb.h, bh = kb.b * p.H + h;
    const int D = p.Dh[h];
    const int We = p.W > 1 ? p.W : 1;
    const bool ends = kb.type == 0;
    const int n_ce = p.T / D;                  // chunk ends of the sequence (all positions: D = 1)
    // query tiles: from the tile holding the block's first key to the last query holding one
    int tq_start, t_end;
    if (ends) {
        tq_start = ((BM * kb.m) * D + D - 1) / BN * BN;
        t_end = p.T;
    } else {
        tq_start = BM * kb.m;
        t_end = min(p.T, BM * kb.m + BM - 1 + We);
    }
    const int nq = (t_end - tq_start + BN - 1) / BN;

    if (threadIdx.x == 0) {
        mbar_init(&sh.kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.qd_full[s], 1);
            mbar_init(&sh.qd_empty[s], 1);
            mbar_init(&sh.sdp_full[s], 1);
            mbar_init(&sh.pds_full[s], 128);
            mbar_init(&sh.kv_done[s], 1);
        }
        mbar_init(&sh.fin, 1);
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(&sh.tmem, 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sh.tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const bool strided = ends && D > 1;
            const CUtensorMap *mk = strided ? &p.tm_kd128[max(p.dslot[h], 0)] : &p.tm_k128;
            const CUtensorMap *mv = strided ? &p.tm_vd128[max(p.dslot[h], 0)] : &p.tm_v128;
            const int row = BM * kb.m;
            tc::prefetch_tmap(mk);
            tc::prefetch_tmap(&p.tm_qh64);
            mbar_arrive_expect_tx(&sh.kv_full, 4 * SUB128);
            tc::tma_load_3d(smem + OFF_K, mk, 0, row, bh, &sh.kv_full);
            tc::tma_load_3d(smem + OFF_K + SUB128, mk, 64, row, bh, &sh.kv_full);
            tc::tma_load_3d(smem + OFF_V, mv, 0, row, bh, &sh.kv_full);
            tc::tma_load_3d(smem + OFF_V + SUB128, mv, 64, row, bh, &sh.kv_full);
            int issued = 0;
            for (int u = 0; u < nq; ++u) {
                const int s = u & 1;
                if (u >= 2 && !wait_bar(&sh.abort, p.hdr, &sh.qd_empty[s], ((u >> 1) - 1) & 1, 8)) break;
                const int tq = tq_start + BN * u;
                uint8_t *qs = smem + OFF_Q + s * 2 * SUB64, *gs = smem + OFF_G + s * 2 * SUB64;
                mbar_arrive_expect_tx(&sh.qd_full[s], 4 * SUB64);
                tc::tma_load_3d(qs, &p.tm_qh64, 0, tq, bh, &sh.qd_full[s]);
                tc::tma_load_3d(qs + SUB64, &p.tm_qh64, 64, tq, bh, &sh.qd_full[s]);
                tc::tma_load_3d(gs, &p.tm_g64, 0, tq, bh, &sh.qd_full[s]);
                tc::tma_load_3d(gs + SUB64, &p.tm_g64, 64, tq, bh, &sh.qd_full[s]);
                issued = u + 1;
            }
            if (sh.abort) {
                for (int u = max(0, issued - 2); u < issued; ++u) wait_drain(&sh.qd_full[u & 1], (u >> 1) & 1);
                wait_drain(&sh.kv_full, 0);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = tc::idesc_bf16(BM, BN, 0);       // Q^^T, dO^T: K-major B
            constexpr uint32_t IDESC_A = tc::idesc_bf16(BM, DHEAD, 1);    // dO, Q^: MN-major B
            const uint32_t sk = smem_u32(smem + OFF_K), sv = smem_u32(smem + OFF_V);
            bool ok = wait_bar(&sh.abort, p.hdr, &sh.kv_full, 0, 9);
            tc::fence_after_sync();
            for (int u = 0; ok && u <= nq; ++u) {
                if (u < nq) {
                    const int s = u & 1;
                    if (!wait_bar(&sh.abort, p.hdr, &sh.qd_full[s], (u >> 1) & 1, 10)) break;
                    // buffers s hold P^T, dS^T of tile u-2 until its dV, dK MMAs have read them
                    if (u >= 2 && !wait_bar(&sh.abort, p.hdr, &sh.kv_done[s], ((u - 2) >> 1) & 1, 11)) break;
                    tc::fence_after_sync();
                    const uint32_t sq = smem_u32(smem + OFF_Q + s * 2 * SUB64);
                    const uint32_t sg = smem_u32(smem + OFF_G + s * 2 * SUB64);
                    for (int kk = 0; kk < DHEAD / 16; ++kk) {
                        const uint32_t ao = (kk >> 2) * SUB128 + (kk & 3) * 32;
                        const uint32_t bo = (kk >> 2) * SUB64 + (kk & 3) * 32;
                        tc::mma_bf16_ss(tmem + COL_S + s * BN, tc::smem_desc_sw128(sk + ao, 16, 1024),
                                        tc::smem_desc_sw128(sq + bo, 16, 1024), IDESC_S, kk > 0);
                        tc::mma_bf16_ss(tmem + COL_P + s * BN, tc::smem_desc_sw128(sv + ao, 16, 1024),
                                        tc::smem_desc_sw128(sg + bo, 16, 1024), IDESC_S, kk > 0);
                    }
                    tc::mma_commit(&sh.sdp_full[s]);
                }
                if (u >= 1) {
                    const int up = u - 1, s = up & 1;
                    if (!wait_bar(&sh.abort, p.hdr, &sh.pds_full[s], (up >> 1) & 1, 12)) break;
                    tc::fence_after_sync();
                    const uint32_t sq = smem_u32(smem + OFF_Q + s * 2 * SUB64);
                    const uint32_t sg = smem_u32(smem + OFF_G + s * 2 * SUB64);
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        const uint32_t boff = kk * 16 * 128;
                        tc::mma_bf16_ts(tmem + COL_V, tmem + COL_S + s * BN + kk * 8,
                                        tc::smem_desc_sw128(sg + boff, SUB64, 1024), IDESC_A,
                                        (up > 0 || kk > 0) ? 1u : 0u);
                        tc::mma_bf16_ts(tmem + COL_K, tmem + COL_P + s * BN + kk * 8,
                                        tc::smem_desc_sw128(sq + boff, SUB64, 1024), IDESC_A,
                                        (up > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&sh.kv_done[s]);
                    tc::mma_commit(&sh.qd_empty[s]);
                }
            }
            tc::mma_commit(&sh.fin);
            wait_drain(&sh.fin, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ P^T, dS^T rows + epilogue
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;           // key row in the block == TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
        // this row's key position and whether this block owns its gradient
        int pos;
        bool own;
        if (ends) {
            const int i = BM * kb.m + r;
            pos = i * D + D - 1;
            own = i < n_ce;
        } else {
            pos = BM * kb.m + r;
            own = pos < p.T && (D == 1 || pos % D != D - 1);
        }
        bool ok = true;
        for (int u = 0; u < nq; ++u) {
            const int s = u & 1;
            const int tq = tq_start + BN * u;
            // lse and Delta of the tile's 64 queries, shared by all rows: lane l holds those of
            // queries tq + l and tq + 32 + l, every lane takes column c by a shuffle
            float lse2[2], dl2[2];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int tt = tq + 32 * hf + lane;
                lse2[hf] = tt < p.T ? p.lse[(size_t)bh * p.T + tt] : 0.f;
                dl2[hf] = tt < p.T ? p.delta[(size_t)bh * p.T + tt] : 0.f;
            }
            if (!__all_sync(0xffffffffu, wait_bar(&sh.abort, p.hdr, &sh.sdp_full[s], (u >> 1) & 1, 13))) { ok = false; break; }
            tc::fence_after_sync();
            float sv[BN], pv[BN];
            tc::tmem_ld32(tl + COL_S + s * BN, reinterpret_cast<uint32_t *>(sv));
            tc::tmem_ld32(tl + COL_S + s * BN + 32, reinterpret_cast<uint32_t *>(sv) + 32);
            tc::tmem_ld32(tl + COL_P + s * BN, reinterpret_cast<uint32_t *>(pv));
            tc::tmem_ld32(tl + COL_P + s * BN + 32, reinterpret_cast<uint32_t *>(pv) + 32);
            tc::tmem_wait_ld();
            // queries t = tq + c holding this key: t >= pos (chunk end), pos <= t < pos + We (other)
            const int c_lo = pos - tq;
            const int c_hi = own ? (ends ? p.T - 1 - tq : min(pos + We - 1, p.T - 1) - tq) : -1;
            uint32_t pp[32], pd[32];
#pragma unroll
            for (int i = 0; i < BN / 2; ++i) {
                float pr[2], d2[2];
#pragma unroll
                for (int u2 = 0; u2 < 2; ++u2) {
                    const int c = 2 * i + u2;
                    const float lc = __shfl_sync(0xffffffffu, lse2[c >> 5], c & 31);
                    const float dc = __shfl_sync(0xffffffffu, dl2[c >> 5], c & 31);
                    pr[u2] = (c >= c_lo && c <= c_hi) ? ex2_approx(fmaf(sv[c], p.scale_log2, -lc)) : 0.f;
                    d2[u2] = pr[u2] * (pv[c] - dc);
                }
                pp[i] = pack_bf16(pr[0], pr[1]);
                pd[i] = pack_bf16(d2[0], d2[1]);
            }
            tc::tmem_st32(tl + COL_S + s * BN, pp);
            tc::tmem_st32(tl + COL_P + s * BN, pd);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            mbar_arrive(&sh.pds_full[s]);
        }
        if (ok && nq > 0)
            ok = __all_sync(0xffffffffu, wait_bar(&sh.abort, p.hdr, &sh.kv_done[(nq - 1) & 1], ((nq - 1) >> 1) & 1, 14));
        if (ok) {
            tc::fence_after_sync();
            const size_t ro = ((size_t)bh * p.T + (own ? pos : 0)) * DHEAD * 2;
            uint8_t *rk = static_cast<uint8_t *>(p.dk) + ro, *rv = static_cast<uint8_t *>(p.dv) + ro;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float xv[32], xk[32];
                if (nq > 0) {
                    tc::tmem_ld32(tl + COL_V + 32 * c, reinterpret_cast<uint32_t *>(xv));
                    tc::tmem_ld32(tl + COL_K + 32 * c, reinterpret_cast<uint32_t *>(xk));
                    tc::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) xv[i] = xk[i] = 0.f;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) xk[i] *= p.scale;
                if (own) {
                    store_row32(rv, 32 * c, xv);
                    store_row32(rk, 32 * c, xk);
                }
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------------------ self keys
// W <= 1: a key j that is not a chunk end is held by query j alone, so its gradients are one
// pair's: p = 2^(scale log2e <q^_j, k~_j> - lse_j), ds = p (<dO_j, v~_j> - Delta_j),
// dk~_j = scale ds q^_j, dv~_j = p dO_j.  One warp per row, four channels per lane.
__global__ void __launch_bounds__(256) attn_bwd_self_kernel(const __grid_constant__ Params p,
                                                            const void *qh, const void *k, const void *v,
                                                            const void *dO) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, h = bh % p.H;
    const int j = blockIdx.x * 8 + warp;
    const int D = p.Dh[h];
    if (j >= p.T || D == 1 || j % D == D - 1) return;
    const size_t off = ((size_t)bh * p.T + j) * DHEAD * 2 + lane * 8;
    auto ld4 = [&](const void *base, float *x) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint8_t *>(base) + off));
        x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    };
    float q[4], kk[4], vv[4], g[4];
    ld4(qh, q);
    ld4(k, kk);
    ld4(v, vv);
    ld4(dO, g);
    float sd = 0.f, pd = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        sd = fmaf(q[i], kk[i], sd);
        pd = fmaf(g[i], vv[i], pd);
    }
    sd = warp_sum(sd);
    pd = warp_sum(pd);
    const size_t r = (size_t)bh * p.T + j;
    const float pr = ex2_approx(fmaf(sd, p.scale_log2, -p.lse[r]));
    const float ds = pr * (pd - p.delta[r]) * p.scale;
    *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.dk) + off) =
        make_uint2(pack_bf16(ds * q[0], ds * q[1]), pack_bf16(ds * q[2], ds * q[3]));
    *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.dv) + off) =
        make_uint2(pack_bf16(pr * g[0], pr * g[1]), pack_bf16(pr * g[2], pr * g[3]));
}

// ------------------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 bwd_encode_fn() {
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

// (d, rows, BH) bf16 view, box (64 channels, box_rows, 1), 128-byte swizzle, zero fill outside.
bool bwd_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t BH, uint64_t row_stride,
             uint64_t slice_stride, uint32_t box_rows) {
    auto fn = bwd_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)DHEAD, rows, BH};
    cuuint64_t strides[2] = {row_stride, slice_stride};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attn_bwd_sm100_supported(const AttnBwdParams &a, int dtype) {
    if (dtype != RAT_BF16 || a.d != DHEAD || a.n_sink != 0 || a.T < 1) return false;
    int dv[kMaxDil], nd = 0;
    for (int h = 0; h < a.H; ++h) {
        const int D = a.Dh[h];
        if (D == 1) continue;
        bool seen = false;
        for (int i = 0; i < nd; ++i) seen |= dv[i] == D;
        if (!seen) {
            if (nd == kMaxDil) return false;
            dv[nd++] = D;
        }
    }
    return true;
}

// The two tensor-core launches of the backward (q^ and Delta already in the workspace, lse
// given or recomputed by the caller).
int launch_attn_bwd_sm100(const AttnBwdParams &a, void *stream) {
    WsHeader *hdr = a.hdr;
    Params p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t BH = (uint64_t)a.B * a.H, T = (uint64_t)a.T;
    const uint64_t row = DHEAD * 2, slice = T * row;
    // dq key blocks: 32 keys (two CTAs per SM) when every head is dilated, else 64
    bool dense = false;
    for (int h = 0; h < a.H; ++h) dense |= a.Dh[h] == 1;
    const uint32_t bnq = dense ? 64 : 32;
    if (!bwd_map(&p.tm_qh128, a.qh, T, BH, row, slice, 128) || !bwd_map(&p.tm_g128, a.dO, T, BH, row, slice, 128) ||
        !bwd_map(&p.tm_qh64, a.qh, T, BH, row, slice, 64) || !bwd_map(&p.tm_g64, a.dO, T, BH, row, slice, 64) ||
        !bwd_map(&p.tm_kq, a.k, T, BH, row, slice, bnq) || !bwd_map(&p.tm_vq, a.v, T, BH, row, slice, bnq) ||
        !bwd_map(&p.tm_k128, a.k, T, BH, row, slice, 128) || !bwd_map(&p.tm_v128, a.v, T, BH, row, slice, 128))
        return RAT_ERR_CUDA;
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
                const uint8_t *kb = static_cast<const uint8_t *>(a.k) + off;
                const uint8_t *vb = static_cast<const uint8_t *>(a.v) + off;
                if (!bwd_map(&p.tm_kdq[slot], kb, cap, BH, (uint64_t)D * row, slice, bnq) ||
                    !bwd_map(&p.tm_vdq[slot], vb, cap, BH, (uint64_t)D * row, slice, bnq) ||
                    !bwd_map(&p.tm_kd128[slot], kb, cap, BH, (uint64_t)D * row, slice, 128) ||
                    !bwd_map(&p.tm_vd128[slot], vb, cap, BH, (uint64_t)D * row, slice, 128))
                    return RAT_ERR_CUDA;
            } else {   // no chunk end inside the sequence: no block reads these maps
                p.tm_kdq[slot] = p.tm_kq;
                p.tm_vdq[slot] = p.tm_vq;
                p.tm_kd128[slot] = p.tm_k128;
                p.tm_vd128[slot] = p.tm_v128;
            }
        }
        p.dslot[h] = slot;
    }
    // heads by dilation, smallest (most keys) first
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
    p.ntiles = (a.T + dqk::BM - 1) / dqk::BM;
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
    const int dq_items = items;
    // dkv sections: chunk-end blocks of every group (longest walks first), then the other keys
    int kitems = 0;
    p.nsec = 0;
    for (int type = 0; type < 2; ++type)
        for (int gi = 0; gi < p.ngroups; ++gi) {
            const int D = a.Dh[order[p.grp_head0[gi]]];
            // (with W <= 1 a key that is not a chunk end has only its own query: the per-row
            // kernel below takes those keys)
            const int nblk = type == 0 ? (a.T / D + dkv::BM - 1) / dkv::BM
                                       : (D > 1 && a.W > 1 ? (a.T + dkv::BM - 1) / dkv::BM : 0);
            if (nblk == 0) continue;
            p.sec_item0[p.nsec] = kitems;
            p.sec_grp[p.nsec] = gi;
            p.sec_type[p.nsec] = type;
            p.sec_nblk[p.nsec] = nblk;
            kitems += nblk * a.B * p.grp_nheads[gi];
            ++p.nsec;
        }
    p.sec_item0[p.nsec] = kitems;
    p.lse = a.lse;
    p.delta = a.delta;
    p.kg = a.k;
    p.vg = a.v;
    p.dq = a.dq;
    p.dk = a.dk;
    p.dv = a.dv;
    p.hdr = hdr;
    p.pos0 = a.pos0;
    p.rope = a.rope;
    p.scale = a.scale;
    p.scale_log2 = a.scale_log2;
    for (int c = 0; c < 64; ++c) p.theta[c] = a.theta[c];

    static std::atomic<uint64_t> attr_q64{0}, attr_q32{0}, attr_k{0};
    int st = bnq == 64
                 ? set_smem_attr(reinterpret_cast<const void *>(attn_bwd_dq_sm100_kernel<64>), DqCfg<64>::SMEM, &attr_q64)
                 : set_smem_attr(reinterpret_cast<const void *>(attn_bwd_dq_sm100_kernel<32>), DqCfg<32>::SMEM, &attr_q32);
    if (st != RAT_OK) return st;
    st = set_smem_attr(reinterpret_cast<const void *>(attn_bwd_dkv_sm100_kernel), dkv::SMEM, &attr_k);
    if (st != RAT_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dq_items > 0) {
        if (bnq == 64) attn_bwd_dq_sm100_kernel<64><<<(unsigned)dq_items, kThreads, DqCfg<64>::SMEM, s>>>(p);
        else attn_bwd_dq_sm100_kernel<32><<<(unsigned)dq_items, kThreads, DqCfg<32>::SMEM, s>>>(p);
    }
    if (kitems > 0) attn_bwd_dkv_sm100_kernel<<<(unsigned)kitems, kThreads, dkv::SMEM, s>>>(p);
    bool self_keys = false;
    for (int h = 0; h < a.H; ++h) self_keys |= a.Dh[h] > 1;
    if (self_keys && a.W <= 1) {
        dim3 grid((unsigned)((a.T + 7) / 8), (unsigned)(a.B * a.H));
        attn_bwd_self_kernel<<<grid, 256, 0, s>>>(p, a.qh, a.k, a.v, a.dO);
    }
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

}  // namespace rat
