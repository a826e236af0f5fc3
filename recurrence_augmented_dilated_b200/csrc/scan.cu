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

// 16 bytes of a row -> VEC floats.
template <typename E> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    static RAT_DEVICE void load(const uint8_t *s, float *x) {
        uint32_t a, b, c, d;
        ld_shared_v4(s, a, b, c, d);
        x[0] = __uint_as_float(a); x[1] = __uint_as_float(b);
        x[2] = __uint_as_float(c); x[3] = __uint_as_float(d);
    }
    static RAT_DEVICE void store(void *g, const float *x) {
        st_global_v4(g, __float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                     __float_as_uint(x[3]));
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    static RAT_DEVICE void load(const uint8_t *s, float *x) {
        uint32_t u[4];
        ld_shared_v4(s, u[0], u[1], u[2], u[3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) { x[2 * i] = bf16_lo(u[i]); x[2 * i + 1] = bf16_hi(u[i]); }
    }
    static RAT_DEVICE void store(void *g, const float *x) {
        st_global_v4(g, pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                     pack_bf16(x[6], x[7]));
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

        // ---- pass 1: gates of this lane's R rows (kept for pass 2) and their aggregate
        float G[R][VEC], OG[R][VEC];
        float A[VEC], Bk[VEC], Bv[VEC];
#pragma unroll
        for (int j = 0; j < VEC; ++j) { A[j] = 1.f; Bk[j] = 0.f; Bv[j] = 0.f; }
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = seg * R + i;
            float xa[VEC], xk[VEC], xv[VEC];
            if (r < rows) {
                const int off = r * C::ROWB + cl * 16;
                Vec<E>::load(sa + off, xa);
                Vec<E>::load(sk + off, xk);
                Vec<E>::load(sv + off, xv);
            } else {        // rows past the end: identity step (g = 1, 1-g = 0)
#pragma unroll
                for (int j = 0; j < VEC; ++j) { xa[j] = 1e30f; xk[j] = 0.f; xv[j] = 0.f; }
            }
#pragma unroll
            for (int j = 0; j < VEC; ++j) {
                forget_gate(xa[j], G[i][j], OG[i][j]);
                A[j] *= G[i][j];
                Bk[j] = fmaf(G[i][j], Bk[j], OG[i][j] * xk[j]);
                Bv[j] = fmaf(G[i][j], Bv[j], OG[i][j] * xv[j]);
            }
        }
        // ---- inclusive scan over the segments of this warp (shuffles)
#pragma unroll
        for (int sh = 1; sh < C::SPW; sh <<= 1) {
#pragma unroll
            for (int j = 0; j < VEC; ++j) {
                const float pA = __shfl_up_sync(0xffffffffu, A[j], sh * LPR);
                const float pK = __shfl_up_sync(0xffffffffu, Bk[j], sh * LPR);
                const float pV = __shfl_up_sync(0xffffffffu, Bv[j], sh * LPR);
                if (segw >= sh) {
                    Bk[j] = fmaf(A[j], pK, Bk[j]);
                    Bv[j] = fmaf(A[j], pV, Bv[j]);
                    A[j] *= pA;
                }
            }
        }
        // exclusive prefix of this segment inside its warp
        float eA[VEC], eK[VEC], eV[VEC];
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            eA[j] = __shfl_up_sync(0xffffffffu, A[j], LPR);
            eK[j] = __shfl_up_sync(0xffffffffu, Bk[j], LPR);
            eV[j] = __shfl_up_sync(0xffffffffu, Bv[j], LPR);
            if (segw == 0) { eA[j] = 1.f; eK[j] = 0.f; eV[j] = 0.f; }
        }
        if (segw == C::SPW - 1) {
#pragma unroll
            for (int j = 0; j < VEC; ++j) {
                const int ch = cl * VEC + j;
                sw[(pwarp * 3 + 0) * DH + ch] = A[j];
                sw[(pwarp * 3 + 1) * DH + ch] = Bk[j];
                sw[(pwarp * 3 + 2) * DH + ch] = Bv[j];
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
                        if (globaltimer_ns() - t_start > p.wait_ns) {
                            record_error(hdr, RAT_ERR_TIMEOUT, 0x200u);
                            alive = false;                  // carry zero; error recorded
                            break;
                        }
                        __nanosleep(20);
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
        float hk[VEC], hv[VEC];
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            const int ch = cl * VEC + j;
            const float wk = sw[(pwarp * 3 + 0) * DH + ch], wv = sw[(pwarp * 3 + 1) * DH + ch];
            hk[j] = fmaf(eA[j], wk, eK[j]);
            hv[j] = fmaf(eA[j], wv, eV[j]);
        }
        float rc[VEC], rs[VEC], sc[VEC], ss[VEC];
        const bool first_half = cl < LPR / 2;
        if (p.rope) {
            const long long pos = p.pos0 + t0 + seg * R;
#pragma unroll
            for (int j = 0; j < VEC; ++j) {
                const int f = (cl * VEC + j) % (DH / 2);
                if (p.rope_f32) rope_cs_f32((int)pos, p.theta_f[f], rc[j], rs[j]);
                else rope_cs(pos, p.theta[f], rc[j], rs[j]);
                sc[j] = p.step_cos[f];
                ss[j] = first_half ? -p.step_sin[f] : p.step_sin[f];
                if (first_half) rs[j] = -rs[j];      // first half: x cos - x' sin
            }
        }
        uint8_t *yk = static_cast<uint8_t *>(p.yk);
        uint8_t *yv = static_cast<uint8_t *>(p.yv);
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = seg * R + i;
            const bool valid = r < rows;
            float xk[VEC], xv[VEC];
            if (valid) {
                const int off = r * C::ROWB + cl * 16;
                Vec<E>::load(sk + off, xk);
                Vec<E>::load(sv + off, xv);
            } else {
#pragma unroll
                for (int j = 0; j < VEC; ++j) { xk[j] = 0.f; xv[j] = 0.f; }
            }
            float ok[VEC];
#pragma unroll
            for (int j = 0; j < VEC; ++j) {
                hk[j] = fmaf(G[i][j], hk[j], OG[i][j] * xk[j]);
                hv[j] = fmaf(G[i][j], hv[j], OG[i][j] * xv[j]);
                ok[j] = hk[j];
            }
            if (p.rope) {       // uniform across the grid: the shuffles see every lane
#pragma unroll
                for (int j = 0; j < VEC; ++j) {
                    const float partner = __shfl_xor_sync(0xffffffffu, hk[j], LPR / 2);
                    ok[j] = fmaf(hk[j], rc[j], partner * rs[j]);
                    // advance the angle by one position: (c + i s) * (cos t + i sin t)
                    const float nc = rc[j] * sc[j] - rs[j] * ss[j];
                    const float ns = rs[j] * sc[j] + rc[j] * ss[j];
                    rc[j] = nc;
                    rs[j] = ns;
                }
            }
            if (valid) {
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
    static bool attr_set = false;   // per process; the attribute is per function
    if (!attr_set) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
            return RAT_ERR_CUDA;
        attr_set = true;
    }
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return RAT_ERR_CUDA;
    }
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
