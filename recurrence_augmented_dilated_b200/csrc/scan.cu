// scan.cu -- full-sequence forget-gate recurrence over keys and values (prefill).
//
// "RAT+ Deep Dive", section 2.1: every token's recurrence state accumulates information from
// the start of the sequence (L = T) through a forget gate g = sigmoid(input-dependent logit),
//     h_t = g_t * h_{t-1} + (1 - g_t) * x_t,       x = k and x = v, same g, per channel,
// and prefill computes it in parallel by an associative scan (section 7.3 table).  The map
// h -> g h + (1-g) x is affine, so a run of steps composes to h -> A h + B with
//     A = prod g,   B = sum_s (prod_{r>s} g_r)(1-g_s) x_s,
// and (A1,B1) then (A2,B2) = (A2 A1, A2 B1 + B2).  This kernel is that scan, in three levels:
//
//   lane     : 8 consecutive rows of one 16-byte channel group, sequentially in registers;
//   CTA      : the row segments of a chunk combined by warp shuffles, then across the 8 warps
//              through shared memory;
//   sequence : chunks of the same (b, h) combined by a decoupled look-back -- each chunk
//              publishes its aggregate (A, Bk, Bv) as soon as it has loaded, then walks back
//              over its predecessors' aggregates until it meets an inclusive state.
//
// Data movement: a chunk is TC rows x d channels of one (b, h), i.e. three contiguous byte
// ranges (a, k, v), fetched with three bulk copies (cp.async.bulk) into shared memory.  The
// kernel is persistent (one CTA per SM) and double-buffered: while a CTA computes one chunk,
// the bulk copies of its next chunk are in flight.  Outputs are written with 16-byte stores,
// 16 lanes covering one 256-byte row.  The HBM stream is 3 reads + 2 writes per element, the
// algorithmic minimum.  The gates of pass 1 stay in registers for pass 2, so each element
// costs one exp2 and one reciprocal on the special-function unit.
//
// Chunk order comes from an atomic ticket (chunk-major: all (b, h) advance together); a CTA
// takes its next ticket before finishing the current chunk, and every predecessor it waits
// for was taken earlier by a resident CTA; each wait is bounded by the caller's limit and
// records RAT_ERR_TIMEOUT instead of hanging.  Flags carry a launch epoch, so the workspace is
// never cleared between launches: the last CTA of a launch resets the tickets and bumps the
// epoch.
#include "common.cuh"

namespace rat {

template <typename E, int DH>
struct ScanCfg {
    static constexpr int EB = sizeof(E);
    static constexpr int VEC = 16 / EB;           // channels per lane (one 16-byte vector)
    static constexpr int LPR = DH / VEC;          // lanes per row
    static constexpr int THREADS = 256;
    static constexpr int NPIPE = 2;               // independent chunk pipelines per CTA
    static constexpr int PT = THREADS / NPIPE;    // threads per pipeline
    static constexpr int PW = PT / 32;            // warps per pipeline
    static constexpr int SEGS = PT / LPR;         // row segments per chunk
    static constexpr int SPW = 32 / LPR;          // segments per warp
    static constexpr int R = 8;                   // rows per segment
    static constexpr int TC = SEGS * R;           // rows per chunk
    static constexpr int ROWB = DH * EB;          // bytes per row
    static constexpr int TILEB = TC * ROWB;       // bytes per tensor per chunk (16 KiB)
    static constexpr int STAGEB = 3 * TILEB;      // a, k, v of one chunk
    static constexpr int SWB = PW * 3 * DH * 4;   // per-warp aggregates, then carries
    static constexpr int PIPEB = 2 * STAGEB + SWB + 2 * DH * 4;   // two stages + sw + state in
    static constexpr int SMEM = NPIPE * PIPEB;
    static_assert(PT >= DH, "one thread per channel in a pipeline");
};

// 16 bytes of a row <-> VEC/2 float pairs (channels 2q, 2q+1 in pair q).
template <typename E> struct Vec;
template <> struct Vec<float> {
    static constexpr int NP = 2;
    static RAT_DEVICE void load(const uint8_t *s, f2_t *x) {
        uint32_t a, b, c, d;
        ld_shared_v4(s, a, b, c, d);
        x[0] = f2(__uint_as_float(a), __uint_as_float(b));
        x[1] = f2(__uint_as_float(c), __uint_as_float(d));
    }
    static RAT_DEVICE void store(void *g, const f2_t *x) {
        st_global_v4(g, __float_as_uint(f2lo(x[0])), __float_as_uint(f2hi(x[0])),
                     __float_as_uint(f2lo(x[1])), __float_as_uint(f2hi(x[1])));
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int NP = 4;
    static RAT_DEVICE void load(const uint8_t *s, f2_t *x) {
        uint32_t u[4];
        ld_shared_v4(s, u[0], u[1], u[2], u[3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = f2_from_bf16x2(u[i]);
    }
    static RAT_DEVICE void store(void *g, const f2_t *x) {
        st_global_v4(g, f2_to_bf16x2(x[0]), f2_to_bf16x2(x[1]), f2_to_bf16x2(x[2]), f2_to_bf16x2(x[3]));
    }
};

// Look-back records: each value is one 64-bit word, (tag << 32) | float bits, written with a
// single relaxed store; a reader accepts a word only when its tag is this launch's tag, so a
// value and its validity always travel together.
RAT_DEVICE uint64_t tagged(uint32_t tag, float v) { return ((uint64_t)tag << 32) | __float_as_uint(v); }

// Wait (bounded) for the tagged word at w; returns false if the wait ran out.
RAT_DEVICE bool wait_word(const uint64_t *w, uint32_t tag, float &v, uint64_t t_start, uint64_t limit_ns,
                          WsHeader *hdr) {
    for (;;) {
        const uint64_t x = ld_relaxed_gpu_u64(w);
        if ((uint32_t)(x >> 32) == tag) {
            v = __uint_as_float((uint32_t)x);
            return true;
        }
        if (globaltimer_ns() - t_start > limit_ns) {
            record_error(hdr, RAT_ERR_TIMEOUT, 0x200u);
            return false;
        }
        __nanosleep(20);
    }
}

template <typename E, int DH>
__global__ void __launch_bounds__(256, 1) recur_kernel(const __grid_constant__ RecurParams p) {
    using C = ScanCfg<E, DH>;
    constexpr int VEC = C::VEC, LPR = C::LPR, R = C::R;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bar[C::NPIPE][2];
    __shared__ int s_ticket[C::NPIPE][2];
    __shared__ uint32_t s_epoch;

    const int tid = threadIdx.x;
    const int pipe = tid / C::PT, pt = tid % C::PT;              // pipeline and thread in it
    const int pwarp = pt >> 5, lane = tid & 31;
    const int seg = pt / LPR, cl = pt % LPR, segw = lane / LPR;
    const int barid = 1 + pipe;                                   // named barrier of this pipeline
    uint8_t *pbase = smem + pipe * C::PIPEB;
    float *sw = reinterpret_cast<float *>(pbase + 2 * C::STAGEB);          // [PW][3][DH]
    float *sH = reinterpret_cast<float *>(pbase + 2 * C::STAGEB + C::SWB); // [2][DH] state in
    WsHeader *hdr = p.hdr;
    const int total = p.BH * p.nchunks;

    // issue the three bulk copies of chunk `ticket` into stage `st` (thread 0 of the pipeline)
    auto load_chunk = [&](int ticket, int st) {
        const int c = ticket / p.BH, bh = ticket % p.BH;
        const int rows = min(C::TC, p.T - c * C::TC);
        const size_t row0 = (size_t)bh * p.T + (size_t)c * C::TC;
        const uint32_t bytes = (uint32_t)rows * C::ROWB;
        uint8_t *s = pbase + st * C::STAGEB;
        mbar_arrive_expect_tx(&bar[pipe][st], 3 * bytes);
        bulk_g2s(s, static_cast<const uint8_t *>(p.a) + row0 * C::ROWB, bytes, &bar[pipe][st]);
        bulk_g2s(s + C::TILEB, static_cast<const uint8_t *>(p.k) + row0 * C::ROWB, bytes, &bar[pipe][st]);
        bulk_g2s(s + 2 * C::TILEB, static_cast<const uint8_t *>(p.v) + row0 * C::ROWB, bytes, &bar[pipe][st]);
    };
    auto pipe_sync = [&]() { asm volatile("bar.sync %0, %1;" :: "r"(barid), "r"(C::PT) : "memory"); };

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

    for (int it = 0;; ++it) {
        const int st = it & 1;
        const int ticket = s_ticket[pipe][st];
        if (ticket >= total) break;
        // prefetch the next chunk into the other stage (consumed by the previous iteration,
        // which ended with a pipeline barrier)
        if (pt == 0) {
            const int nt = (int)atomicAdd(&hdr->ticket, 1u);
            s_ticket[pipe][st ^ 1] = nt;
            if (nt < total) load_chunk(nt, st ^ 1);
        }
        const int c = ticket / p.BH, bh = ticket % p.BH;     // chunk-major order
        const int t0 = c * C::TC;
        const int rows = min(C::TC, p.T - t0);
        const size_t chunk_id = (size_t)bh * p.nchunks + c;
        const size_t row0 = (size_t)bh * p.T + t0;
        const bool publish = c != p.fault_chunk;            // false only under the test hook
        const uint8_t *sa = pbase + st * C::STAGEB, *sk = sa + C::TILEB, *sv = sa + 2 * C::TILEB;
        mbar_wait_bounded(&bar[pipe][st], (it >> 1) & 1, hdr, 0x100u);

        // ---- pass 1: gates of this lane's R rows (kept for pass 2) and their aggregate, on
        // packed float pairs (channels 2q, 2q+1)
        constexpr int NP = VEC / 2;
        const f2_t kOne2 = f2(1.f, 1.f), kZero2 = f2(0.f, 0.f);
        f2_t G[R][NP], OG[R][NP];
        f2_t A[NP], Bk[NP], Bv[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) { A[q] = kOne2; Bk[q] = kZero2; Bv[q] = kZero2; }
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = seg * R + i;
            const int rr = r < rows ? r : rows - 1;          // rows past the end: identity step
            const int off = rr * C::ROWB + cl * 16;
            f2_t xa[NP], xk[NP], xv[NP];
            Vec<E>::load(sa + off, xa);
            Vec<E>::load(sk + off, xk);
            Vec<E>::load(sv + off, xv);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                forget_gate2(xa[q], G[i][q], OG[i][q]);
                if (r >= rows) { G[i][q] = kOne2; OG[i][q] = kZero2; }
                A[q] = f2_mul(A[q], G[i][q]);
                Bk[q] = f2_fma(G[i][q], Bk[q], f2_mul(OG[i][q], xk[q]));
                Bv[q] = f2_fma(G[i][q], Bv[q], f2_mul(OG[i][q], xv[q]));
            }
        }
        // ---- inclusive scan over the segments of this warp (shuffles)
#pragma unroll
        for (int sh = 1; sh < C::SPW; sh <<= 1) {
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const f2_t pA = f2(__shfl_up_sync(0xffffffffu, f2lo(A[q]), sh * LPR),
                                   __shfl_up_sync(0xffffffffu, f2hi(A[q]), sh * LPR));
                const f2_t pK = f2(__shfl_up_sync(0xffffffffu, f2lo(Bk[q]), sh * LPR),
                                   __shfl_up_sync(0xffffffffu, f2hi(Bk[q]), sh * LPR));
                const f2_t pV = f2(__shfl_up_sync(0xffffffffu, f2lo(Bv[q]), sh * LPR),
                                   __shfl_up_sync(0xffffffffu, f2hi(Bv[q]), sh * LPR));
                if (segw >= sh) {
                    Bk[q] = f2_fma(A[q], pK, Bk[q]);
                    Bv[q] = f2_fma(A[q], pV, Bv[q]);
                    A[q] = f2_mul(A[q], pA);
                }
            }
        }
        // exclusive prefix of this segment inside its warp
        f2_t eA[NP], eK[NP], eV[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            eA[q] = f2(__shfl_up_sync(0xffffffffu, f2lo(A[q]), LPR), __shfl_up_sync(0xffffffffu, f2hi(A[q]), LPR));
            eK[q] = f2(__shfl_up_sync(0xffffffffu, f2lo(Bk[q]), LPR), __shfl_up_sync(0xffffffffu, f2hi(Bk[q]), LPR));
            eV[q] = f2(__shfl_up_sync(0xffffffffu, f2lo(Bv[q]), LPR), __shfl_up_sync(0xffffffffu, f2hi(Bv[q]), LPR));
            if (segw == 0) { eA[q] = kOne2; eK[q] = kZero2; eV[q] = kZero2; }
        }
        if (segw == C::SPW - 1) {
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const int ch = cl * VEC + 2 * q;
                sw[(pwarp * 3 + 0) * DH + ch] = f2lo(A[q]);
                sw[(pwarp * 3 + 0) * DH + ch + 1] = f2hi(A[q]);
                sw[(pwarp * 3 + 1) * DH + ch] = f2lo(Bk[q]);
                sw[(pwarp * 3 + 1) * DH + ch + 1] = f2hi(Bk[q]);
                sw[(pwarp * 3 + 2) * DH + ch] = f2lo(Bv[q]);
                sw[(pwarp * 3 + 2) * DH + ch + 1] = f2hi(Bv[q]);
            }
        }
        pipe_sync();

        // ---- one thread per channel: chunk aggregate (published), look-back for the state
        // entering the chunk, inclusive state (published), carries entering each warp
        if (pt < DH) {
            const int ch = pt;
            float cA = 1.f, cK = 0.f, cV = 0.f;
#pragma unroll
            for (int w = 0; w < C::PW; ++w) {
                const float a = sw[(w * 3 + 0) * DH + ch];
                cK = fmaf(a, cK, sw[(w * 3 + 1) * DH + ch]);
                cV = fmaf(a, cV, sw[(w * 3 + 2) * DH + ch]);
                cA *= a;
            }
            if (c > 0 && publish) {
                uint64_t *agg = p.agg + chunk_id * 3 * DH;
                st_relaxed_gpu_u64(agg + ch, tagged(tag, cA));
                st_relaxed_gpu_u64(agg + DH + ch, tagged(tag, cK));
                st_relaxed_gpu_u64(agg + 2 * DH + ch, tagged(tag, cV));
            }
            float Hk = 0.f, Hv = 0.f;     // state entering this chunk
            if (c == 0) {
                if (p.h0k) Hk = p.h0k[(size_t)bh * DH + ch];
                if (p.h0v) Hv = p.h0v[(size_t)bh * DH + ch];
            } else {
                float xA = 1.f, xK = 0.f, xV = 0.f;   // composition of chunks j+1 .. c-1
                const uint64_t t_start = globaltimer_ns();
                uint32_t spins = 0;
                bool alive = true;
                for (int j = c - 1; j >= 0 && alive; --j) {
                    const size_t jid = (size_t)bh * p.nchunks + j;
                    const uint64_t *pj = p.pre + jid * 2 * DH;
                    const uint64_t *aj = p.agg + jid * 3 * DH;
                    // predecessor j: its inclusive state if published, else its aggregate
                    for (;;) {
                        const uint64_t x = ld_relaxed_gpu_u64(pj + ch);
                        if ((uint32_t)(x >> 32) == tag) {
                            float hv;
                            alive = wait_word(pj + DH + ch, tag, hv, t_start, p.wait_ns, hdr);
                            Hk = fmaf(xA, __uint_as_float((uint32_t)x), xK);
                            Hv = fmaf(xA, hv, xV);
                            j = -1;                         // done
                            break;
                        }
                        const uint64_t y = ld_relaxed_gpu_u64(aj + ch);
                        if ((uint32_t)(y >> 32) == tag) {
                            float bk, bv;
                            alive = wait_word(aj + DH + ch, tag, bk, t_start, p.wait_ns, hdr) &&
                                    wait_word(aj + 2 * DH + ch, tag, bv, t_start, p.wait_ns, hdr);
                            xK = fmaf(xA, bk, xK);
                            xV = fmaf(xA, bv, xV);
                            xA *= __uint_as_float((uint32_t)y);
                            break;                          // next predecessor
                        }
                        if ((++spins & 7u) == 0u && globaltimer_ns() - t_start > p.wait_ns) {
                            record_error(hdr, RAT_ERR_TIMEOUT, 0x200u);
                            alive = false;                  // carry zero; error recorded
                            break;
                        }
                        __nanosleep(32);
                    }
                }
            }
            const float outK = fmaf(cA, Hk, cK), outV = fmaf(cA, Hv, cV);
            if (publish) {
                uint64_t *pre = p.pre + chunk_id * 2 * DH;
                st_relaxed_gpu_u64(pre + ch, tagged(tag, outK));
                st_relaxed_gpu_u64(pre + DH + ch, tagged(tag, outV));
            }
            if (c == p.nchunks - 1) {
                if (p.hTk) p.hTk[(size_t)bh * DH + ch] = outK;
                if (p.hTv) p.hTv[(size_t)bh * DH + ch] = outV;
            }
            float hK = Hk, hV = Hv;
#pragma unroll
            for (int w = 0; w < C::PW; ++w) {
                const float a = sw[(w * 3 + 0) * DH + ch];
                const float bk = sw[(w * 3 + 1) * DH + ch];
                const float bv = sw[(w * 3 + 2) * DH + ch];
                sw[(w * 3 + 0) * DH + ch] = hK;
                sw[(w * 3 + 1) * DH + ch] = hV;
                hK = fmaf(a, hK, bk);
                hV = fmaf(a, hV, bv);
            }
        }
        pipe_sync();

        // ---- pass 2: rerun the recurrence from the carry with the kept gates; write k~
        // (optionally rotated) and v~
        f2_t hk[NP], hv[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            const int ch = cl * VEC + 2 * q;
            const f2_t wk = f2(sw[(pwarp * 3 + 0) * DH + ch], sw[(pwarp * 3 + 0) * DH + ch + 1]);
            const f2_t wv = f2(sw[(pwarp * 3 + 1) * DH + ch], sw[(pwarp * 3 + 1) * DH + ch + 1]);
            hk[q] = f2_fma(eA[q], wk, eK[q]);
            hv[q] = f2_fma(eA[q], wv, eV[q]);
        }
        // RoPE: rotation (rc + i rs) of this lane's channels at its first row, advanced one
        // position per row by (sc + i ss); the first half of the channels takes x cos - x' sin
        f2_t rc[NP], rs[NP], sc[NP], ss[NP], nss[NP];
        const bool first_half = cl < LPR / 2;
        if (p.rope) {
            const long long pos = p.pos0 + t0 + seg * R;
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                float c2[2], s2[2], a2[2], b2[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int f = (cl * VEC + 2 * q + u) % (DH / 2);
                    if (p.rope_f32) rope_cs_f32((int)pos, p.theta_f[f], c2[u], s2[u]);
                    else rope_cs(pos, p.theta[f], c2[u], s2[u]);
                    a2[u] = p.step_cos[f];
                    b2[u] = first_half ? -p.step_sin[f] : p.step_sin[f];
                    if (first_half) s2[u] = -s2[u];
                }
                rc[q] = f2(c2[0], c2[1]);
                rs[q] = f2(s2[0], s2[1]);
                sc[q] = f2(a2[0], a2[1]);
                ss[q] = f2(b2[0], b2[1]);
                nss[q] = f2(-b2[0], -b2[1]);
            }
        }
        uint8_t *yk = static_cast<uint8_t *>(p.yk);
        uint8_t *yv = static_cast<uint8_t *>(p.yv);
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = seg * R + i;
            const int rr = r < rows ? r : rows - 1;
            const int off = rr * C::ROWB + cl * 16;
            f2_t xk[NP], xv[NP];
            Vec<E>::load(sk + off, xk);
            Vec<E>::load(sv + off, xv);
            f2_t ok[NP];
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                hk[q] = f2_fma(G[i][q], hk[q], f2_mul(OG[i][q], xk[q]));
                hv[q] = f2_fma(G[i][q], hv[q], f2_mul(OG[i][q], xv[q]));
                ok[q] = hk[q];
            }
            if (p.rope) {       // uniform across the grid: the shuffles see every lane
#pragma unroll
                for (int q = 0; q < NP; ++q) {
                    const f2_t partner = f2(__shfl_xor_sync(0xffffffffu, f2lo(hk[q]), LPR / 2),
                                            __shfl_xor_sync(0xffffffffu, f2hi(hk[q]), LPR / 2));
                    ok[q] = f2_fma(hk[q], rc[q], f2_mul(partner, rs[q]));
                    // advance one position: (c + i s)(cos t + i sin t)
                    const f2_t nc = f2_fma(rc[q], sc[q], f2_mul(rs[q], nss[q]));
                    rs[q] = f2_fma(rs[q], sc[q], f2_mul(rc[q], ss[q]));
                    rc[q] = nc;
                }
            }
            if (r < rows) {
                const size_t go = (row0 + r) * C::ROWB + cl * 16;
                Vec<E>::store(yk + go, ok);
                Vec<E>::store(yv + go, hv);
            }
        }
        pipe_sync();     // this stage's smem and sw are free for the next chunk
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

int recur_chunk_rows(int d, int dtype) {
    const int eb = dtype == RAT_F32 ? 4 : 2;
    return (128 / (d * eb / 16)) * 8;      // (threads per pipeline / lanes per row) x 8 rows
}

size_t recur_workspace_bytes(int BH, int T, int d, int dtype) {
    const size_t tc = (size_t)recur_chunk_rows(d, dtype);
    const size_t nch = (size_t)BH * ((T + tc - 1) / tc);
    return sizeof(WsHeader) + align256(nch * 3 * d * 8) + align256(nch * 2 * d * 8);
}

template <typename E, int DH>
static int launch_one(const RecurParams &p, void *stream) {
    using C = ScanCfg<E, DH>;
    auto kern = recur_kernel<E, DH>;
    static uint64_t attr_done = 0;
    const int st = set_smem_attr(reinterpret_cast<const void *>(kern), C::SMEM, &attr_done);
    if (st != RAT_OK) return st;
    const int sms = current_sm_count();
    if (sms <= 0) return RAT_ERR_CUDA;
    // persistent: one CTA per SM, each walking chunks in ticket order
    const long long total = (long long)p.BH * p.nchunks;
    const unsigned grid = (unsigned)(total < sms ? total : sms);
    kern<<<grid, C::THREADS, C::SMEM, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

int launch_recur(const RecurParams &p, int dtype, void *stream) {
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
