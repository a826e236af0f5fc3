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
// Written with the carry c_t = g_{t+1} mu_{t+1} that enters row t from the right, each row is
// the affine map c_{t-1} = g_t (c_t + e_t) of its own row's data (c_{T-1} = dL/dh_{T-1},
// mu_t = e_t + c_t, dh0 = c_{-1}), so a run of rows composes to c -> A c + B like the forward
// step, and the backward is the forward scan's structure run from the end of the sequence:
//
//   lane     : R consecutive rows of four channels, last row first, in registers;
//   CTA      : the row segments of a chunk combined by warp shuffles, then across the warps of
//              a pipeline through shared memory;
//   sequence : chunks of one (b, h) combined by a decoupled look-back to the right -- each
//              chunk publishes its map (A, Bk, Bv) as soon as its data has been read, then walks
//              over the chunks after it until it meets a published carry.
//
// Data movement: a chunk is TC rows of one (b, h) (64 rows for bf16, 32 for float32; R rows per
// lane keep the second pass's prefetched rows within the registers); a, dk~ and dv~ come
// by three bulk copies into shared memory (double-buffered, the next chunk's copies in flight
// while one is computed) and serve both passes; the second pass reads k, v and the forward
// outputs of the row before each row straight from global memory, issued before the look-back
// so that they arrive while it runs.  HBM traffic: seven reads and three writes per element, the
// minimum.
//
// The chunk-local form (RESET; RAT's recurrence restarted before every absolute position that
// is a multiple of L) cuts the recurrence at block starts: nothing passes from a block start t
// to t - 1 (the row's map becomes c -> 0), the state entering a block start is 0 in da, and h0
// gets a gradient only when row 0 is not a block start.
//
// Chunk order comes from an atomic ticket, last chunks first, so the chunks a look-back waits for
// were taken earlier by resident CTAs; every wait is bounded (RAT_ERR_TIMEOUT recorded in the
// workspace) and the records carry a launch tag, so the workspace is never cleared between calls.
#include "common.cuh"

namespace rat {

namespace {

template <typename E, int DH>
struct BwdCfg {
    static constexpr int EB = sizeof(E);
    static constexpr int LPR = DH / 4;            // lanes per row: four channels (two pairs) each
    static constexpr int HALFB = DH / 2 * EB;     // byte offset of the second half of a row
    static constexpr int THREADS = 512;
    static constexpr int NPIPE = 2;               // independent chunk pipelines per CTA
    static constexpr int PT = THREADS / NPIPE;
    static constexpr int PW = PT / 32;
    static constexpr int SEGS = PT / LPR;         // row segments per chunk
    static constexpr int SPW = 32 / LPR;          // segments per warp
    static constexpr int ROWB = DH * EB;
    static constexpr int TC = EB == 2 ? 64 : 32;  // rows per chunk
    static constexpr int TILEB = TC * ROWB;       // bytes per tensor per chunk (8 or 16 KiB)
    static constexpr int R = TC / SEGS;           // rows per segment
    static constexpr int LBW = 2;                 // chunks read per look-back round
    static constexpr int STAGEB = 3 * TILEB;      // a, dk~, dv~ of one chunk
    static constexpr int SWB = PW * 3 * DH * 4;   // per-warp maps, then carries
    static constexpr int PIPEB = 2 * STAGEB + SWB;
    static constexpr int SMEM = NPIPE * PIPEB;
    static_assert(PT >= DH, "one thread per channel in a pipeline");
    static_assert(R * SEGS == TC && R >= 1, "whole segments per chunk");
};

// A lane's four channels of one row, as loaded (converted to float pairs when used).
template <typename E> struct LaneRaw;
template <> struct LaneRaw<__nv_bfloat16> {
    uint32_t lo, hi;
    template <int HALFB>
    RAT_DEVICE void load(const uint8_t *row, int l) {
        lo = __ldg(reinterpret_cast<const unsigned int *>(row + 4 * l));
        hi = __ldg(reinterpret_cast<const unsigned int *>(row + HALFB + 4 * l));
    }
    RAT_DEVICE void get(f2_t *x) const {
        x[0] = f2_from_bf16x2(lo);
        x[1] = f2_from_bf16x2(hi);
    }
};
template <> struct LaneRaw<float> {
    uint2 lo, hi;
    template <int HALFB>
    RAT_DEVICE void load(const uint8_t *row, int l) {
        lo = __ldg(reinterpret_cast<const uint2 *>(row + 8 * l));
        hi = __ldg(reinterpret_cast<const uint2 *>(row + HALFB + 8 * l));
    }
    RAT_DEVICE void get(f2_t *x) const {
        x[0] = f2(__uint_as_float(lo.x), __uint_as_float(lo.y));
        x[1] = f2(__uint_as_float(hi.x), __uint_as_float(hi.y));
    }
};

// the transposed rotation of a lane's pairs: (x1, x2) -> (x1 c + x2 s, x2 c - x1 s)
RAT_DEVICE void rot_t(const f2_t *y, f2_t c, f2_t s, f2_t *x) {
    const f2_t ns = f2_mul(s, f2(-1.f, -1.f));
    x[0] = f2_fma(y[1], s, f2_mul(y[0], c));
    x[1] = f2_fma(y[0], ns, f2_mul(y[1], c));
}

// one step back in position: angle - theta
RAT_DEVICE void step_back(f2_t &c, f2_t &s, f2_t sc, f2_t ss) {
    const f2_t ns = f2_mul(ss, f2(-1.f, -1.f));
    const f2_t nc = f2_fma(s, ss, f2_mul(c, sc));
    s = f2_fma(c, ns, f2_mul(s, sc));
    c = nc;
}

// Look-back records: (tag << 32) | float bits in one 64-bit word, valid only with this launch's tag
RAT_DEVICE uint64_t tagged(uint32_t tag, float v) { return ((uint64_t)tag << 32) | __float_as_uint(v); }

}  // namespace

template <typename E, int DH, bool RESET>
__global__ void __launch_bounds__(BwdCfg<E, DH>::THREADS, 1) bwd_scan_kernel(const __grid_constant__ RecurBwdParams p) {
    using C = BwdCfg<E, DH>;
    constexpr int LPR = C::LPR, R = C::R, HALF = DH / 2, NP = 2;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bar[C::NPIPE][2];
    __shared__ int s_ticket[C::NPIPE][2];
    __shared__ uint32_t s_epoch;
    __shared__ float s_theta_f[HALF], s_step_c[HALF], s_step_s[HALF];
    __shared__ double s_theta[HALF];

    const int tid = threadIdx.x;
    const int pipe = tid / C::PT, pt = tid % C::PT;              // pipeline and thread in it
    const int pwarp = pt >> 5, lane = tid & 31;
    const int seg = pt / LPR, cl = pt % LPR, segw = lane / LPR;
    const int chq[NP] = {2 * cl, 2 * cl + HALF};                   // first channel of each pair
    const int barid = 1 + pipe;                                   // named barrier of this pipeline
    uint8_t *pbase = smem + pipe * C::PIPEB;
    float *sw = reinterpret_cast<float *>(pbase + 2 * C::STAGEB);          // [PW][3][DH]
    WsHeader *hdr = p.hdr;
    const int total = p.BH * p.nch;

    // ticket -> (chunk, b*h): chunk-major from the last chunk, so a chunk's right neighbours
    // always hold earlier tickets
    auto chunk_of = [&](int ticket, int &c, int &bh) {
        c = p.nch - 1 - ticket / p.BH;
        bh = ticket % p.BH;
    };
    // the three bulk copies (a, dk~, dv~) of chunk `ticket` into stage `st` (thread 0 of the pipeline)
    auto load_chunk = [&](int ticket, int st) {
        int c, bh;
        chunk_of(ticket, c, bh);
        const int rows = min(C::TC, p.T - c * C::TC);
        const size_t row0 = (size_t)bh * p.T + (size_t)c * C::TC;
        const uint32_t bytes = (uint32_t)rows * C::ROWB;
        uint8_t *s = pbase + st * C::STAGEB;
        mbar_arrive_expect_tx(&bar[pipe][st], 3 * bytes);
        bulk_g2s(s, static_cast<const uint8_t *>(p.a) + row0 * C::ROWB, bytes, &bar[pipe][st]);
        bulk_g2s(s + C::TILEB, static_cast<const uint8_t *>(p.dyk) + row0 * C::ROWB, bytes, &bar[pipe][st]);
        bulk_g2s(s + 2 * C::TILEB, static_cast<const uint8_t *>(p.dyv) + row0 * C::ROWB, bytes, &bar[pipe][st]);
    };
    auto pipe_sync = [&]() { asm volatile("bar.sync %0, %1;" :: "r"(barid), "r"(C::PT) : "memory"); };
    // one look-back round of channel `ch` of (b, h) = bh: the chunks j, j+1, ..., j+LBW-1
    // (clamped at the last), each its carry (k, v) and its map (A, Bk, Bv)
    auto read_window = [&](int bh, int j, int ch, uint64_t (&w)[C::LBW][5]) {
#pragma unroll
        for (int u = 0; u < C::LBW; ++u) {
            const size_t jid = (size_t)bh * p.nch + min(j + u, p.nch - 1);
            const uint64_t *pj = p.pre + jid * 2 * DH + ch;
            const uint64_t *aj = p.agg + jid * 3 * DH + ch;
            w[u][0] = ld_relaxed_gpu_u64(pj);
            w[u][1] = ld_relaxed_gpu_u64(pj + DH);
            w[u][2] = ld_relaxed_gpu_u64(aj);
            w[u][3] = ld_relaxed_gpu_u64(aj + DH);
            w[u][4] = ld_relaxed_gpu_u64(aj + 2 * DH);
        }
    };
    // (cos, sin) of this lane's two frequencies at position pos0 + t
    auto lane_angle = [&](long long t, f2_t &c, f2_t &s) {
        float c2[2], s2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int f = 2 * cl + u;
            const long long pos = p.pos0 + t;
            if (p.rope_f32) rope_cs_f32((int)pos, s_theta_f[f], c2[u], s2[u]);
            else rope_cs(pos, s_theta[f], c2[u], s2[u]);
        }
        c = f2(c2[0], c2[1]);
        s = f2(s2[0], s2[1]);
    };
    auto block_start = [&](long long t) { return (p.pos0 + t) % p.reset == 0; };

    if (tid < HALF) {           // RoPE tables, read per lane below without divergent constant loads
        s_theta_f[tid] = p.theta_f[tid];
        s_theta[tid] = p.theta[tid];
        s_step_c[tid] = p.step_cos[tid];
        s_step_s[tid] = p.step_sin[tid];
    }
    if (tid == 0) {
        s_epoch = *reinterpret_cast<volatile uint32_t *>(&hdr->epoch);
        for (int q = 0; q < C::NPIPE; ++q) {
            mbar_init(&bar[q][0], 1);
            mbar_init(&bar[q][1], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();
    const uint32_t epoch_raw = s_epoch;
    const uint32_t tag = (epoch_raw & 0x7fffffffu) | 0x80000000u;   // never 0: a zeroed workspace never matches
    if (pt == 0) {
        const int t0k = (int)atomicAdd(&hdr->ticket, 1u);
        s_ticket[pipe][0] = t0k;
        if (t0k < total) load_chunk(t0k, 0);
    }
    pipe_sync();

    const f2_t kOne2 = f2(1.f, 1.f), kZero2 = f2(0.f, 0.f), kNegOne2 = f2(-1.f, -1.f);
    f2_t sc = kOne2, ss = kZero2;                 // one-position rotation of this lane's frequencies
    if (p.rope) {
        sc = f2(s_step_c[2 * cl], s_step_c[2 * cl + 1]);
        ss = f2(s_step_s[2 * cl], s_step_s[2 * cl + 1]);
    }

    for (int it = 0;; ++it) {
        const int st = it & 1;
        const int ticket = s_ticket[pipe][st];
        if (ticket >= total) break;
        if (pt == 0) {          // prefetch the next chunk into the other stage
            const int nt = (int)atomicAdd(&hdr->ticket, 1u);
            s_ticket[pipe][st ^ 1] = nt;
            if (nt < total) load_chunk(nt, st ^ 1);
        }
        int c, bh;
        chunk_of(ticket, c, bh);
        const int t0 = c * C::TC;
        const int rows = min(C::TC, p.T - t0);
        const size_t chunk_id = (size_t)bh * p.nch + c;
        const size_t base = (size_t)bh * p.T * C::ROWB;
        const bool publish = c != p.fault_chunk;            // false only under the test hook
        const uint8_t *sa = pbase + st * C::STAGEB, *sdk = sa + C::TILEB, *sdv = sa + 2 * C::TILEB;
        const int r_top = seg * R + R - 1;                  // this lane's last row in the chunk
        const bool last = c == p.nch - 1;
        // nothing enters the chunk from the right when its right neighbour starts a block
        const bool cut = RESET && !last && block_start(t0 + C::TC);
        // chunk-local form: bit i of rmask marks row seg*R + i as the first of a block
        uint32_t rmask = 0;
        if (RESET) {
            const long long m = (p.pos0 + t0 + seg * R) % p.reset;
            const long long off = m == 0 ? 0 : p.reset - m;               // rows to the next block start
            const int lim = min(R, rows - seg * R);                        // this segment's rows
            if (off < lim) {
                const int step = p.reset < R ? (int)p.reset : R;          // beyond R: one start at most
#pragma unroll 1
                for (int i = (int)off; i < lim; i += step) rmask |= 1u << i;
            }
        }
        mbar_wait_bounded(&bar[pipe][st], (it >> 1) & 1, hdr, 0x300u);

        // ---- pass 1: this lane's rows, last first, composed into (A, Bk, Bv): c_out = A c_in + B
        f2_t A[NP], Bk[NP], Bv[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) { A[q] = kOne2; Bk[q] = kZero2; Bv[q] = kZero2; }
        {
            f2_t rc = kOne2, rs = kZero2;
            if (p.rope) lane_angle(t0 + r_top, rc, rs);
#pragma unroll
            for (int i = R - 1; i >= 0; --i) {
                const int r = seg * R + i;
                const bool valid = r < rows;                // rows past the end: identity map
                const int off = (valid ? r : rows - 1) * C::ROWB;
                f2_t xa[NP], yk[NP], yv[NP];
                Lane<E>::template load<C::HALFB>(sa + off, cl, xa);
                Lane<E>::template load<C::HALFB>(sdk + off, cl, yk);
                Lane<E>::template load<C::HALFB>(sdv + off, cl, yv);
                f2_t ek[NP] = {yk[0], yk[1]};
                if (p.rope) {
                    rot_t(yk, rc, rs, ek);
                    step_back(rc, rs, sc, ss);
                }
                const bool start = RESET && ((rmask >> i) & 1u);
                if (valid) {
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        const f2_t g = forget_gate2(xa[q]);
                        A[q] = start ? kZero2 : f2_mul(g, A[q]);
                        Bk[q] = start ? kZero2 : f2_mul(g, f2_add(Bk[q], ek[q]));
                        Bv[q] = start ? kZero2 : f2_mul(g, f2_add(Bv[q], yv[q]));
                    }
                }
            }
        }
        // the second pass's global rows (k_t, v_t and the forward outputs at t - 1), in flight
        // during the look-back
        LaneRaw<E> gk[R], gv[R], hk[R], hv[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = min(seg * R + i, rows - 1);
            const int tp = max(t0 + r - 1, 0);      // row 0's predecessor is h0 (set below)
            gk[i].template load<C::HALFB>(static_cast<const uint8_t *>(p.k) + base + (size_t)(t0 + r) * C::ROWB, cl);
            gv[i].template load<C::HALFB>(static_cast<const uint8_t *>(p.v) + base + (size_t)(t0 + r) * C::ROWB, cl);
            hk[i].template load<C::HALFB>(static_cast<const uint8_t *>(p.yk) + base + (size_t)tp * C::ROWB, cl);
            hv[i].template load<C::HALFB>(static_cast<const uint8_t *>(p.yv) + base + (size_t)tp * C::ROWB, cl);
        }

        // ---- suffix scan over the segments of this warp (shuffles): the map from the warp's
        // right edge to the left edge of each segment
#pragma unroll
        for (int sh = 1; sh < C::SPW; sh <<= 1) {
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const f2_t pA = f2(__shfl_down_sync(0xffffffffu, f2lo(A[q]), sh * LPR),
                                   __shfl_down_sync(0xffffffffu, f2hi(A[q]), sh * LPR));
                const f2_t pK = f2(__shfl_down_sync(0xffffffffu, f2lo(Bk[q]), sh * LPR),
                                   __shfl_down_sync(0xffffffffu, f2hi(Bk[q]), sh * LPR));
                const f2_t pV = f2(__shfl_down_sync(0xffffffffu, f2lo(Bv[q]), sh * LPR),
                                   __shfl_down_sync(0xffffffffu, f2hi(Bv[q]), sh * LPR));
                if (segw + sh < C::SPW) {   // this segment's map applied after the later ones
                    Bk[q] = f2_fma(A[q], pK, Bk[q]);
                    Bv[q] = f2_fma(A[q], pV, Bv[q]);
                    A[q] = f2_mul(A[q], pA);
                }
            }
        }
        // the map from the warp's right edge to this segment's right edge (exclusive suffix)
        f2_t eA[NP], eK[NP], eV[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            if (C::SPW > 1) {
                eA[q] = f2(__shfl_down_sync(0xffffffffu, f2lo(A[q]), LPR), __shfl_down_sync(0xffffffffu, f2hi(A[q]), LPR));
                eK[q] = f2(__shfl_down_sync(0xffffffffu, f2lo(Bk[q]), LPR), __shfl_down_sync(0xffffffffu, f2hi(Bk[q]), LPR));
                eV[q] = f2(__shfl_down_sync(0xffffffffu, f2lo(Bv[q]), LPR), __shfl_down_sync(0xffffffffu, f2hi(Bv[q]), LPR));
            }
            if (C::SPW == 1 || segw == C::SPW - 1) { eA[q] = kOne2; eK[q] = kZero2; eV[q] = kZero2; }
        }
        if (segw == 0) {         // the whole warp's map
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const int ch = chq[q];
                sw[(pwarp * 3 + 0) * DH + ch] = f2lo(A[q]);
                sw[(pwarp * 3 + 0) * DH + ch + 1] = f2hi(A[q]);
                sw[(pwarp * 3 + 1) * DH + ch] = f2lo(Bk[q]);
                sw[(pwarp * 3 + 1) * DH + ch + 1] = f2hi(Bk[q]);
                sw[(pwarp * 3 + 2) * DH + ch] = f2lo(Bv[q]);
                sw[(pwarp * 3 + 2) * DH + ch + 1] = f2hi(Bv[q]);
            }
        }
        pipe_sync();

        // ---- one thread per channel: the chunk's map (published), the look-back for the carry
        // entering the chunk from the right, the carry leaving it (published), and the carries
        // entering each warp
        if (pt < DH) {
            const int ch = pt;
            float cA = 1.f, cK = 0.f, cV = 0.f;
#pragma unroll
            for (int wp = C::PW - 1; wp >= 0; --wp) {
                const float a = sw[(wp * 3 + 0) * DH + ch];
                cK = fmaf(a, cK, sw[(wp * 3 + 1) * DH + ch]);
                cV = fmaf(a, cV, sw[(wp * 3 + 2) * DH + ch]);
                cA *= a;
            }
            if (!last && publish) {
                uint64_t *agg = p.agg + chunk_id * 3 * DH;
                st_relaxed_gpu_u64(agg + ch, tagged(tag, cA));
                st_relaxed_gpu_u64(agg + DH + ch, tagged(tag, cK));
                st_relaxed_gpu_u64(agg + 2 * DH + ch, tagged(tag, cV));
            }
            float Ck = 0.f, Cv = 0.f;     // carry entering the chunk's last row
            if (last) {
                if (p.dhTk) Ck = p.dhTk[(size_t)bh * DH + ch];
                if (p.dhTv) Cv = p.dhTv[(size_t)bh * DH + ch];
            } else if (cut) {
                // the next chunk starts a block: nothing passes into this one
            } else {
                // Walk forward from j = c + 1, C::LBW chunks per round, all five words of each read
                // at once: a chunk with its carry ends the walk, one with only its map is composed
                // in and passed, one with neither stops the round and the next round re-reads from
                // there.
                float xA = 1.f, xK = 0.f, xV = 0.f;   // composition of chunks c+1 .. j-1
                const uint64_t t_start = globaltimer_ns();
                uint32_t spins = 0;
                int j = c + 1;
                for (;;) {
                    uint64_t w[C::LBW][5];
                    read_window(bh, j, ch, w);
                    bool done = false, stop = false;
                    int passed = 0;
#pragma unroll
                    for (int u = 0; u < C::LBW; ++u) {
                        if (done || stop || j + u >= p.nch) continue;
                        auto ok = [&](int e) { return (uint32_t)(w[u][e] >> 32) == tag; };
                        auto val = [&](int e) { return __uint_as_float((uint32_t)w[u][e]); };
                        if (ok(0) && ok(1)) {
                            Ck = fmaf(xA, val(0), xK);
                            Cv = fmaf(xA, val(1), xV);
                            done = true;
                        } else if (ok(2) && ok(3) && ok(4)) {
                            xK = fmaf(xA, val(3), xK);
                            xV = fmaf(xA, val(4), xV);
                            xA *= val(2);
                            ++passed;
                            if (RESET && xA == 0.f) {   // a block starts in between: nothing further passes
                                Ck = xK;
                                Cv = xV;
                                done = true;
                            }
                        } else {
                            stop = true;
                        }
                    }
                    if (done) break;
                    j += passed;
                    if (passed == 0) {
                        if ((++spins & 7u) == 0u && globaltimer_ns() - t_start > p.wait_ns) {
                            record_error(hdr, RAT_ERR_TIMEOUT, 0x400u);
                            break;                          // carry zero; error recorded
                        }
                        __nanosleep(32);
                    }
                }
            }
            const float outK = fmaf(cA, Ck, cK), outV = fmaf(cA, Cv, cV);   // c_{t0 - 1}
            if (publish) {
                uint64_t *pre = p.pre + chunk_id * 2 * DH;
                st_relaxed_gpu_u64(pre + ch, tagged(tag, outK));
                st_relaxed_gpu_u64(pre + DH + ch, tagged(tag, outV));
            }
            if (c == 0) {               // dh0 = g_0 mu_0 = c_{-1}
                if (p.dh0k) p.dh0k[(size_t)bh * DH + ch] = outK;
                if (p.dh0v) p.dh0v[(size_t)bh * DH + ch] = outV;
            }
            float hK = Ck, hV = Cv;
#pragma unroll
            for (int wp = C::PW - 1; wp >= 0; --wp) {
                const float a = sw[(wp * 3 + 0) * DH + ch];
                const float bk = sw[(wp * 3 + 1) * DH + ch];
                const float bv = sw[(wp * 3 + 2) * DH + ch];
                sw[(wp * 3 + 0) * DH + ch] = hK;
                sw[(wp * 3 + 1) * DH + ch] = hV;
                hK = fmaf(a, hK, bk);
                hV = fmaf(a, hV, bv);
            }
        }
        pipe_sync();

        // ---- pass 2: from the carry entering this segment, rows last first: mu = e + c, the
        // outputs, then the carry g mu for the row before
        f2_t ck[NP], cv[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            const int ch = chq[q];
            const f2_t wk = f2(sw[(pwarp * 3 + 0) * DH + ch], sw[(pwarp * 3 + 0) * DH + ch + 1]);
            const f2_t wv = f2(sw[(pwarp * 3 + 1) * DH + ch], sw[(pwarp * 3 + 1) * DH + ch + 1]);
            ck[q] = f2_fma(eA[q], wk, eK[q]);
            cv[q] = f2_fma(eA[q], wv, eV[q]);
        }
        // rotation at t (for dk~_t) and at t - 1 (for k~_{t-1})
        f2_t rc = kOne2, rs = kZero2, pc = kOne2, ps = kZero2;
        if (p.rope) {
            lane_angle(t0 + r_top, rc, rs);
            pc = rc;
            ps = rs;
            step_back(pc, ps, sc, ss);
        }
        f2_t h0k[NP] = {kZero2, kZero2}, h0v[NP] = {kZero2, kZero2};
        if (t0 == 0 && seg == 0) {
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const size_t o = (size_t)bh * DH + chq[q];
                if (p.h0k) h0k[q] = f2(p.h0k[o], p.h0k[o + 1]);
                if (p.h0v) h0v[q] = f2(p.h0v[o], p.h0v[o + 1]);
            }
        }
        uint8_t *odk = static_cast<uint8_t *>(p.dk) + base;
        uint8_t *odv = static_cast<uint8_t *>(p.dv) + base;
        uint8_t *oda = static_cast<uint8_t *>(p.da) + base;
#pragma unroll
        for (int i = R - 1; i >= 0; --i) {
            const int r = seg * R + i;
            const int t = t0 + r;
            if (r < rows) {
                const int off = r * C::ROWB;
                f2_t xa[NP], yk[NP], yv[NP], xk[NP], xv[NP], hkr[NP], hpv[NP];
                Lane<E>::template load<C::HALFB>(sa + off, cl, xa);
                Lane<E>::template load<C::HALFB>(sdk + off, cl, yk);
                Lane<E>::template load<C::HALFB>(sdv + off, cl, yv);
                gk[i].get(xk);
                gv[i].get(xv);
                hk[i].get(hkr);
                hv[i].get(hpv);
                f2_t ek[NP] = {yk[0], yk[1]}, hpk[NP] = {hkr[0], hkr[1]};
                if (p.rope) {
                    rot_t(yk, rc, rs, ek);
                    rot_t(hkr, pc, ps, hpk);
                }
                if (t == 0) {
#pragma unroll
                    for (int q = 0; q < NP; ++q) { hpk[q] = h0k[q]; hpv[q] = h0v[q]; }
                }
                const bool start = RESET && ((rmask >> i) & 1u);
                if (start) {                               // the state entering a block start is 0
#pragma unroll
                    for (int q = 0; q < NP; ++q) { hpk[q] = kZero2; hpv[q] = kZero2; }
                }
                f2_t ok[NP], ov[NP], oa[NP];
#pragma unroll
                for (int q = 0; q < NP; ++q) {
                    const f2_t muk = f2_add(ek[q], ck[q]);
                    const f2_t muv = f2_add(yv[q], cv[q]);
                    const f2_t g = forget_gate2(xa[q]);
                    const f2_t og = gate_complement2(g);
                    ok[q] = f2_mul(og, muk);
                    ov[q] = f2_mul(og, muv);
                    const f2_t dk = f2_fma(xk[q], kNegOne2, hpk[q]);     // h_{t-1} - x_t
                    const f2_t dv = f2_fma(xv[q], kNegOne2, hpv[q]);
                    oa[q] = f2_mul(f2_mul(g, og), f2_fma(muk, dk, f2_mul(muv, dv)));
                    ck[q] = start ? kZero2 : f2_mul(g, muk);
                    cv[q] = start ? kZero2 : f2_mul(g, muv);
                }
                const size_t o = (size_t)t * C::ROWB;
                Lane<E>::template store<C::HALFB>(odk + o, cl, ok);
                Lane<E>::template store<C::HALFB>(odv + o, cl, ov);
                Lane<E>::template store<C::HALFB>(oda + o, cl, oa);
            }
            if (p.rope) {
                rc = pc;
                rs = ps;
                step_back(pc, ps, sc, ss);
            }
        }
        pipe_sync();     // this stage's shared memory and sw are free for the next chunk
    }

    // ---- launch bookkeeping: the last pipeline resets the ticket counter and bumps the epoch
    if (pt == 0) {
        __threadfence();
        if (atomicAdd(&hdr->done, 1u) == gridDim.x * C::NPIPE - 1) {
            hdr->ticket = 0;
            hdr->done = 0;
            __threadfence();
            atomicExch(&hdr->epoch, epoch_raw + 1u);
        }
    }
}

int recur_bwd_chunk_rows(int d, int dtype) {
    (void)d;
    return dtype == RAT_F32 ? 32 : 64;     // BwdCfg<E, d>::TC
}

size_t recur_bwd_workspace_bytes(int BH, int T, int d) {
    // sized for the shortest chunks (float32), so that one size serves both dtypes
    const size_t tc = (size_t)recur_bwd_chunk_rows(d, RAT_F32);
    const size_t nch = (size_t)BH * (((size_t)T + tc - 1) / tc);
    return sizeof(WsHeader) + align256(nch * 3 * d * 8) + align256(nch * 2 * d * 8);
}

template <typename E, int DH>
static int launch_bwd_one(const RecurBwdParams &p, cudaStream_t s) {
    using C = BwdCfg<E, DH>;
    auto kern = p.reset > 0 ? bwd_scan_kernel<E, DH, true> : bwd_scan_kernel<E, DH, false>;
    static std::atomic<uint64_t> attr_done[2] = {{0}, {0}};
    const int st = set_smem_attr(reinterpret_cast<const void *>(kern), C::SMEM, &attr_done[p.reset > 0]);
    if (st != RAT_OK) return st;
    const int sms = current_sm_count();
    if (sms <= 0) return RAT_ERR_CUDA;
    // persistent: one CTA per SM, each walking chunks in ticket order
    const long long total = (long long)p.BH * p.nch;
    const unsigned grid = (unsigned)(total < sms ? total : sms);
    kern<<<grid, C::THREADS, C::SMEM, s>>>(p);
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
