// scan.cu -- full-sequence forget-gate recurrence over keys and values (prefill).
//
// "RAT+ Deep Dive", section 2.1: the recurrence of RAT+ runs over the whole sequence (L = T), so a
// token's state sums up everything before it, decayed by a forget gate g = sigmoid(logit) that
// depends on the input:
//     h_t = g_t * h_{t-1} + (1 - g_t) * x_t,       x = k and x = v, same g, per channel,
// and prefill computes it in parallel by an associative scan (section 7.3 table).  The map
// h -> g h + (1-g) x is affine, so a run of steps composes to h -> A h + B with
//     A = prod g,   B = sum_s (prod_{r>s} g_r)(1-g_s) x_s,
// and (A1,B1) then (A2,B2) = (A2 A1, A2 B1 + B2).  This kernel is that scan, in three levels:
//
//   lane     : R consecutive rows of four channels, sequentially in registers;
//   CTA      : the row segments of a chunk combined by warp shuffles, then across the warps
//              of a pipeline through shared memory;
//   sequence : chunks of the same (b, h) combined by a decoupled look-back -- each chunk
//              publishes its aggregate (A, Bk, Bv) as soon as it has loaded, then walks back
//              over its predecessors' aggregates until it meets an inclusive state.
//
// Lane layout: lane l of a row holds the channel pairs (2l, 2l+1) and (2l + d/2, 2l+1 + d/2).
// The two pairs are each other's rotate-half RoPE partners, so the rotation of k~ needs no
// data from other lanes, and every shared-memory load and global store of a warp touches one
// contiguous run of bytes.
//
// Data movement: a chunk is TC rows x d channels of one (b, h), i.e. three contiguous byte
// ranges (a, k, v) of 16 KiB, fetched with three bulk copies (cp.async.bulk) into shared
// memory.  The kernel is persistent (one CTA per SM, two independent chunk pipelines) and
// double-buffered: while a pipeline computes one chunk, the bulk copies of its next chunk are
// in flight.  The HBM stream is 3 reads + 2 writes per element, the algorithmic minimum.  The
// gates of pass 1 stay in registers for pass 2, so each element costs one exp2 and one
// reciprocal on the special-function unit.
//
// Chunk order comes from an atomic ticket (chunk-major: all (b, h) advance together); a CTA
// takes its next ticket before finishing the current chunk, and every predecessor it waits
// for was taken earlier by a resident CTA; each wait is bounded by the caller's limit and
// records RAT_ERR_TIMEOUT instead of hanging.  Flags carry a launch epoch, so the workspace is
// never cleared between launches: the last CTA of a launch resets the tickets and bumps the
// epoch.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "tc.cuh"

namespace rat {

template <typename E, int DH>
struct ScanCfg {
    static constexpr int EB = sizeof(E);
    static constexpr int LPR = DH / 4;            // lanes per row: four channels (two pairs) each
    static constexpr int HALFB = DH / 2 * EB;     // byte offset of the second half of a row
    static constexpr int THREADS = 512;
    static constexpr int NPIPE = 2;               // independent chunk pipelines per CTA
    static constexpr int PT = THREADS / NPIPE;    // threads per pipeline
    static constexpr int PW = PT / 32;            // warps per pipeline
    static constexpr int SEGS = PT / LPR;         // row segments per chunk
    static constexpr int SPW = 32 / LPR;          // segments per warp
    static constexpr int ROWB = DH * EB;          // bytes per row
    static constexpr int TILEB = 16384;           // bytes per tensor per chunk
    static constexpr int TC = TILEB / ROWB;       // rows per chunk
    static constexpr int R = TC / SEGS;           // rows per segment
    static constexpr int LBW = 2;                 // predecessors read per look-back round
    static constexpr int STAGEB = 3 * TILEB;      // a, k, v of one chunk
    static constexpr int SWB = PW * 3 * DH * 4;   // per-warp aggregates, then carries
    static constexpr int PIPEB = 2 * STAGEB + SWB;
    static constexpr int SMEM = NPIPE * PIPEB;
    static_assert(PT >= DH, "one thread per channel in a pipeline");
    static_assert(R * SEGS == TC && R >= 1, "whole segments per chunk");
};

// Look-back records: each value is one 64-bit word, (tag << 32) | float bits, written with a
// single relaxed store; a reader accepts a word only when its tag is this launch's tag, so a
// value and its validity always travel together.
RAT_DEVICE uint64_t tagged(uint32_t tag, float v) { return ((uint64_t)tag << 32) | __float_as_uint(v); }

// RESET: the chunk-local form (p.reset > 0) is a separate instantiation, so the full-sequence
// scan carries none of its per-row tests.
template <typename E, int DH, bool RESET>
__global__ void __launch_bounds__(ScanCfg<E, DH>::THREADS, 1) recur_kernel(const __grid_constant__ RecurParams p) {
    using C = ScanCfg<E, DH>;
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
    // one look-back round of channel `ch` of (b, h) = bh: predecessors j, j-1, ..., j-LBW+1
    // (clamped at 0), each its inclusive state (k, v) and its aggregate (A, Bk, Bv)
    auto read_window = [&](int bh, int j, int ch, uint64_t (&w)[C::LBW][5]) {
#pragma unroll
        for (int u = 0; u < C::LBW; ++u) {
            const size_t jid = (size_t)bh * p.nchunks + max(j - u, 0);
            const uint64_t *pj = p.pre + jid * 2 * DH + ch;
            const uint64_t *aj = p.agg + jid * 3 * DH + ch;
            w[u][0] = ld_relaxed_gpu_u64(pj);
            w[u][1] = ld_relaxed_gpu_u64(pj + DH);
            w[u][2] = ld_relaxed_gpu_u64(aj);
            w[u][3] = ld_relaxed_gpu_u64(aj + DH);
            w[u][4] = ld_relaxed_gpu_u64(aj + 2 * DH);
        }
    };

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
        // chunk-local recurrence: bit i of rmask marks row seg*R + i as the first of a block
        // (the carried state is dropped there); a chunk that starts a block needs no carry
        uint32_t rmask = 0;
        bool fresh = false;
        if (RESET) {
            const long long m = (p.pos0 + t0 + seg * R) % p.reset;
            const long long off = m == 0 ? 0 : p.reset - m;               // rows to the next block start
            const int lim = min(R, rows - seg * R);       // rows past the end keep the identity step
            if (off < lim) {
                const int step = p.reset < R ? (int)p.reset : R;          // beyond R: one start at most
#pragma unroll 1
                for (int i = (int)off; i < lim; i += step) rmask |= 1u << i;
            }
            fresh = (p.pos0 + t0) % p.reset == 0;
        }
        // the first look-back round is issued now and consumed after pass 1, so its memory
        // latency overlaps the wait for the data and pass 1
        uint64_t w[C::LBW][5];
        if (pt < DH && c > 0 && !fresh) read_window(bh, c - 1, pt, w);
        mbar_wait_bounded(&bar[pipe][st], (it >> 1) & 1, hdr, 0x100u);

        // ---- pass 1: gates of this lane's R rows (kept for pass 2) and their aggregate
        const f2_t kOne2 = f2(1.f, 1.f), kZero2 = f2(0.f, 0.f);
        f2_t G[R][NP];           // gates; 1 - g is re-formed where it is used
        f2_t A[NP], Bk[NP], Bv[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) { A[q] = kOne2; Bk[q] = kZero2; Bv[q] = kZero2; }
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = seg * R + i;
            const int off = (r < rows ? r : rows - 1) * C::ROWB;   // rows past the end: identity step
            f2_t xa[NP], xk[NP], xv[NP];
            Lane<E>::template load<C::HALFB>(sa + off, cl, xa);
            Lane<E>::template load<C::HALFB>(sk + off, cl, xk);
            Lane<E>::template load<C::HALFB>(sv + off, cl, xv);
            if (RESET && ((rmask >> i) & 1)) {        // a block starts at this row: the state before it is dropped
#pragma unroll
                for (int q = 0; q < NP; ++q) { A[q] = kZero2; Bk[q] = kZero2; Bv[q] = kZero2; }
            }
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                G[i][q] = r < rows ? forget_gate2(xa[q]) : kOne2;
                const f2_t og = gate_complement2(G[i][q]);
                A[q] = f2_mul(A[q], G[i][q]);
                Bk[q] = f2_fma(G[i][q], Bk[q], f2_mul(og, xk[q]));
                Bv[q] = f2_fma(G[i][q], Bv[q], f2_mul(og, xv[q]));
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
            if (C::SPW > 1) {
                eA[q] = f2(__shfl_up_sync(0xffffffffu, f2lo(A[q]), LPR), __shfl_up_sync(0xffffffffu, f2hi(A[q]), LPR));
                eK[q] = f2(__shfl_up_sync(0xffffffffu, f2lo(Bk[q]), LPR), __shfl_up_sync(0xffffffffu, f2hi(Bk[q]), LPR));
                eV[q] = f2(__shfl_up_sync(0xffffffffu, f2lo(Bv[q]), LPR), __shfl_up_sync(0xffffffffu, f2hi(Bv[q]), LPR));
            }
            if (C::SPW == 1 || segw == 0) { eA[q] = kOne2; eK[q] = kZero2; eV[q] = kZero2; }
        }
        if (segw == C::SPW - 1) {
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

        // ---- one thread per channel: chunk aggregate (published), look-back for the state
        // entering the chunk, inclusive state (published), carries entering each warp
        if (pt < DH) {
            const int ch = pt;
            float cA = 1.f, cK = 0.f, cV = 0.f;
#pragma unroll
            for (int wp = 0; wp < C::PW; ++wp) {
                const float a = sw[(wp * 3 + 0) * DH + ch];
                cK = fmaf(a, cK, sw[(wp * 3 + 1) * DH + ch]);
                cV = fmaf(a, cV, sw[(wp * 3 + 2) * DH + ch]);
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
            } else if (fresh) {
                // the chunk starts a block: the state before it is dropped, nothing to wait for
            } else {
                // Walk back from j = c - 1, C::LBW predecessors per round: all five words of each
                // (inclusive state k, v; aggregate A, Bk, Bv) are read at once, so a round costs one
                // memory latency.  A predecessor with its inclusive state ends the walk; one with
                // only its aggregate is composed in and passed; one with neither stops the round,
                // and the next round re-reads from there.
                float xA = 1.f, xK = 0.f, xV = 0.f;   // composition of chunks j+1 .. c-1
                const uint64_t t_start = globaltimer_ns();
                uint32_t spins = 0;
                int j = c - 1;
                for (bool first = true;; first = false) {
                    if (!first) read_window(bh, j, ch, w);      // round 0 was read before pass 1
                    bool done = false, stop = false;
                    int passed = 0;
#pragma unroll
                    for (int u = 0; u < C::LBW; ++u) {
                        if (done || stop || j - u < 0) continue;
                        auto ok = [&](int e) { return (uint32_t)(w[u][e] >> 32) == tag; };
                        auto val = [&](int e) { return __uint_as_float((uint32_t)w[u][e]); };
                        if (ok(0) && ok(1)) {
                            Hk = fmaf(xA, val(0), xK);
                            Hv = fmaf(xA, val(1), xV);
                            done = true;
                        } else if (ok(2) && ok(3) && ok(4)) {
                            xK = fmaf(xA, val(3), xK);
                            xV = fmaf(xA, val(4), xV);
                            xA *= val(2);
                            ++passed;
                            if (RESET && xA == 0.f) {   // a block starts in between: older state is dropped
                                Hk = xK;
                                Hv = xV;
                                done = true;
                            }
                        } else {
                            stop = true;
                        }
                    }
                    if (done) break;
                    j -= passed;
                    if (passed == 0) {
                        if ((++spins & 7u) == 0u && globaltimer_ns() - t_start > p.wait_ns) {
                            record_error(hdr, RAT_ERR_TIMEOUT, 0x200u);
                            break;                          // carry zero; error recorded
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
            for (int wp = 0; wp < C::PW; ++wp) {
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

        // ---- pass 2: rerun the recurrence from the carry with the kept gates; write k~
        // (optionally rotated) and v~
        f2_t hk[NP], hv[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            const int ch = chq[q];
            const f2_t wk = f2(sw[(pwarp * 3 + 0) * DH + ch], sw[(pwarp * 3 + 0) * DH + ch + 1]);
            const f2_t wv = f2(sw[(pwarp * 3 + 1) * DH + ch], sw[(pwarp * 3 + 1) * DH + ch + 1]);
            hk[q] = f2_fma(eA[q], wk, eK[q]);
            hv[q] = f2_fma(eA[q], wv, eV[q]);
        }
        // RoPE: angle (rc, rs) of frequencies 2cl, 2cl+1 at this segment's first row, advanced one
        // position per row by the rotation (sc, ss).  Pair 0 (first half) takes
        // x cos - x' sin, pair 1 (second half) x' cos + x sin.
        f2_t rc = kOne2, rs = kZero2, sc = kOne2, ss = kZero2, nss = kZero2;
        if (p.rope) {
            const long long pos = p.pos0 + t0 + seg * R;
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
        const f2_t kNegOne2 = f2(-1.f, -1.f);
        uint8_t *yk = static_cast<uint8_t *>(p.yk);
        uint8_t *yv = static_cast<uint8_t *>(p.yv);
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = seg * R + i;
            const int off = (r < rows ? r : rows - 1) * C::ROWB;
            f2_t xk[NP], xv[NP];
            Lane<E>::template load<C::HALFB>(sk + off, cl, xk);
            Lane<E>::template load<C::HALFB>(sv + off, cl, xv);
            if (RESET && ((rmask >> i) & 1)) {
#pragma unroll
                for (int q = 0; q < NP; ++q) { hk[q] = kZero2; hv[q] = kZero2; }
            }
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const f2_t og = gate_complement2(G[i][q]);
                hk[q] = f2_fma(G[i][q], hk[q], f2_mul(og, xk[q]));
                hv[q] = f2_fma(G[i][q], hv[q], f2_mul(og, xv[q]));
            }
            f2_t ok[NP] = {hk[0], hk[1]};
            if (p.rope) {
                const f2_t nrs = f2_mul(rs, kNegOne2);
                ok[0] = f2_fma(hk[1], nrs, f2_mul(hk[0], rc));
                ok[1] = f2_fma(hk[0], rs, f2_mul(hk[1], rc));
                // advance one position: (c + i s)(cos t + i sin t)
                const f2_t nc = f2_fma(rc, sc, f2_mul(rs, nss));
                rs = f2_fma(rs, sc, f2_mul(rc, ss));
                rc = nc;
            }
            if (r < rows) {
                const size_t go = (row0 + r) * C::ROWB;
                Lane<E>::template store<C::HALFB>(yk + go, cl, ok);
                Lane<E>::template store<C::HALFB>(yv + go, cl, hv);
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

// ---------------------------------------------------------------------------------------------
// Channel-sliced form (bf16, d = 128, full-sequence recurrence, T a multiple of 16).  The
// channels are independent, so every (b, h) splits into two slices of 64 channels that scan
// separately: slice s holds channels [32s, 32s + 32) and their rotate-half partners
// [64 + 32s, 96 + 32s).  At the same bytes per chunk (48 KiB of a, k, v) a chunk then spans 128
// rows, so each slice's look-back chain advances half as often as the full-row chain of 64-row
// chunks, and the chain -- one L2 round trip per link under the streaming load -- stops setting
// the pace.
//
// Lanes: lane l of warp w holds channels 2c, 2c+1 (c = l mod 16) of the slice's first half and
// their two partners, for the rows of segment 2w + l/16 (8 rows each, 16 segments per chunk),
// so the RoPE rotation needs nothing from other lanes, as in the full-row scan.  Shared memory
// layout: the chunk arrives as one TMA box per tensor from a 5-D view of the tensor,
//     (channel x < 64, segment-in-warp u < 2, half y < 2, row-in-segment i < 8, 16-row group g)
// at byte 2x + 2048u + 128y + 256i + 4096g, box (32, 2, 2, 8, 8); the box lands with u inside
// y, so for each i the two half-warps of a warp read bytes 64 apart, and every load of a warp
// covers all 32 banks once.
struct SliceCfg {
    static constexpr int DH = 128, SC = 64;       // channels per row, per slice
    static constexpr int THREADS = 512, NPIPE = 2, PT = THREADS / NPIPE, PW = PT / 32;
    static constexpr int TC = 128;                // rows per chunk
    static constexpr int R = 8;                   // rows per segment
    static constexpr int SEGS = TC / R;           // two per warp
    static constexpr int TILEB = TC * SC * 2;     // 16 KiB per tensor per chunk
    static constexpr int STAGEB = 3 * TILEB;
    static constexpr int SWB = PW * 3 * SC * 4;   // per-warp aggregates, then carries
    static constexpr int PIPEB = 2 * STAGEB + SWB;
    static constexpr int SMEM = NPIPE * PIPEB + 128;   // + alignment slack for the TMA boxes
    static constexpr int LBW = 2;                 // predecessors read per look-back round
    static_assert(SEGS == 2 * PW && PT >= SC, "two segments per warp, one thread per slice channel");
};

struct SliceParams {
    RecurParams r;              // nchunks counts 128-row chunks here
    CUtensorMap tm_a, tm_k, tm_v;
};

RAT_DEVICE void tma_load_5d(void *smem_dst, const CUtensorMap *map, int c0, int c1, int c2, int c3, int c4,
                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];"
        :: "r"(smem_u32(smem_dst)), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(bar))
        : "memory");
}

__global__ void __launch_bounds__(SliceCfg::THREADS, 1) recur_slice_kernel(const __grid_constant__ SliceParams sp) {
    using C = SliceCfg;
    const RecurParams &p = sp.r;
    constexpr int R = C::R, SC = C::SC, NP = 2;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint64_t bar[C::NPIPE][2];
    __shared__ int s_ticket[C::NPIPE][2];
    __shared__ uint32_t s_epoch;
    __shared__ float s_theta_f[64], s_step_c[64], s_step_s[64];
    __shared__ double s_theta[64];

    const int tid = threadIdx.x;
    const int pipe = tid / C::PT, pt = tid % C::PT;
    const int pwarp = pt >> 5, lane = tid & 31;
    const int segw = lane >> 4, cl = lane & 15;                // segment in the warp, pair in the half
    const int seg = 2 * pwarp + segw;
    const int barid = 1 + pipe;
    uint8_t *smem_al = smem + ((128u - (smem_u32(smem) & 127u)) & 127u);
    uint8_t *pbase = smem_al + pipe * C::PIPEB;
    float *sw = reinterpret_cast<float *>(pbase + 2 * C::STAGEB);          // [PW][3][SC]
    WsHeader *hdr = p.hdr;
    const int items = 2 * p.BH;                                // (b, h, slice)
    const int total = items * p.nchunks;
    // shared-memory byte offset of row r of the chunk, first-half pair of this lane
    auto soff = [&](int r) { return 2048 * (r >> 4) + 256 * (r & 7) + 64 * ((r >> 3) & 1) + 4 * cl; };

    auto load_chunk = [&](int ticket, int st) {
        const int c = ticket / items, item = ticket % items;
        const int g = ((item >> 1) * p.T + c * C::TC) / 16;
        uint8_t *s = pbase + st * C::STAGEB;
        mbar_arrive_expect_tx(&bar[pipe][st], 3 * C::TILEB);
        tma_load_5d(s, &sp.tm_a, 32 * (item & 1), 0, 0, 0, g, &bar[pipe][st]);
        tma_load_5d(s + C::TILEB, &sp.tm_k, 32 * (item & 1), 0, 0, 0, g, &bar[pipe][st]);
        tma_load_5d(s + 2 * C::TILEB, &sp.tm_v, 32 * (item & 1), 0, 0, 0, g, &bar[pipe][st]);
    };
    auto pipe_sync = [&]() { asm volatile("bar.sync %0, %1;" :: "r"(barid), "r"(C::PT) : "memory"); };
    auto read_window = [&](int item, int j, int ch, uint64_t (&w)[C::LBW][5]) {
#pragma unroll
        for (int u = 0; u < C::LBW; ++u) {
            const size_t jid = (size_t)item * p.nchunks + max(j - u, 0);
            const uint64_t *pj = p.pre + jid * 2 * SC + ch;
            const uint64_t *aj = p.agg + jid * 3 * SC + ch;
            w[u][0] = ld_relaxed_gpu_u64(pj);
            w[u][1] = ld_relaxed_gpu_u64(pj + SC);
            w[u][2] = ld_relaxed_gpu_u64(aj);
            w[u][3] = ld_relaxed_gpu_u64(aj + SC);
            w[u][4] = ld_relaxed_gpu_u64(aj + 2 * SC);
        }
    };

    if (tid < 64) {
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
        tc::prefetch_tmap(&sp.tm_a);
        tc::prefetch_tmap(&sp.tm_k);
        tc::prefetch_tmap(&sp.tm_v);
    }
    __syncthreads();
    const uint32_t epoch_raw = s_epoch;
    const uint32_t tag = (epoch_raw & 0x7fffffffu) | 0x80000000u;
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
        if (pt == 0) {
            const int nt = (int)atomicAdd(&hdr->ticket, 1u);
            s_ticket[pipe][st ^ 1] = nt;
            if (nt < total) load_chunk(nt, st ^ 1);
        }
        const int c = ticket / items, item = ticket % items;       // chunk-major order
        const int bh = item >> 1, slice = item & 1;
        const int t0 = c * C::TC;
        const int rows = min(C::TC, p.T - t0);
        const size_t chunk_id = (size_t)item * p.nchunks + c;
        const size_t row0 = (size_t)bh * p.T + t0;
        const bool publish = c != p.fault_chunk;
        const uint8_t *sa = pbase + st * C::STAGEB, *sk = sa + C::TILEB, *sv = sa + 2 * C::TILEB;
        uint64_t w[C::LBW][5];
        if (pt < SC && c > 0) read_window(item, c - 1, pt, w);
        mbar_wait_bounded(&bar[pipe][st], (it >> 1) & 1, hdr, 0x100u);

        // ---- pass 1: gates of this lane's R rows (kept for pass 2) and their aggregate
        const f2_t kOne2 = f2(1.f, 1.f), kZero2 = f2(0.f, 0.f);
        f2_t G[R][NP];
        f2_t A[NP], Bk[NP], Bv[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) { A[q] = kOne2; Bk[q] = kZero2; Bv[q] = kZero2; }
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = seg * R + i;
            const int off = soff(r < rows ? r : rows - 1);         // rows past the end: identity step
            f2_t xa[NP], xk[NP], xv[NP];
            Lane<__nv_bfloat16>::template load<128>(sa + off - 4 * cl, cl, xa);
            Lane<__nv_bfloat16>::template load<128>(sk + off - 4 * cl, cl, xk);
            Lane<__nv_bfloat16>::template load<128>(sv + off - 4 * cl, cl, xv);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                G[i][q] = r < rows ? forget_gate2(xa[q]) : kOne2;
                const f2_t og = gate_complement2(G[i][q]);
                A[q] = f2_mul(A[q], G[i][q]);
                Bk[q] = f2_fma(G[i][q], Bk[q], f2_mul(og, xk[q]));
                Bv[q] = f2_fma(G[i][q], Bv[q], f2_mul(og, xv[q]));
            }
        }
        // ---- the warp's second segment composes the first into its aggregate; the first
        // segment's aggregate is the second's exclusive prefix
        f2_t eA[NP], eK[NP], eV[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            eA[q] = f2(__shfl_up_sync(0xffffffffu, f2lo(A[q]), 16), __shfl_up_sync(0xffffffffu, f2hi(A[q]), 16));
            eK[q] = f2(__shfl_up_sync(0xffffffffu, f2lo(Bk[q]), 16), __shfl_up_sync(0xffffffffu, f2hi(Bk[q]), 16));
            eV[q] = f2(__shfl_up_sync(0xffffffffu, f2lo(Bv[q]), 16), __shfl_up_sync(0xffffffffu, f2hi(Bv[q]), 16));
            if (segw == 0) { eA[q] = kOne2; eK[q] = kZero2; eV[q] = kZero2; }
        }
        if (segw == 1) {
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const f2_t wA = f2_mul(A[q], eA[q]);
                const f2_t wK = f2_fma(A[q], eK[q], Bk[q]);
                const f2_t wV = f2_fma(A[q], eV[q], Bv[q]);
                float2 *s2 = reinterpret_cast<float2 *>(sw) + cl + 16 * q;   // slice channels 2cl (+32q)
                s2[((pwarp * 3 + 0) * SC) / 2] = make_float2(f2lo(wA), f2hi(wA));
                s2[((pwarp * 3 + 1) * SC) / 2] = make_float2(f2lo(wK), f2hi(wK));
                s2[((pwarp * 3 + 2) * SC) / 2] = make_float2(f2lo(wV), f2hi(wV));
            }
        }
        pipe_sync();

        // ---- one thread per slice channel: chunk aggregate (published), look-back for the
        // state entering the chunk, inclusive state (published), carries entering each warp
        if (pt < SC) {
            const int ch = pt;                                     // slice channel
            const int gch = (ch < 32 ? 0 : 64) + 32 * slice + (ch & 31);   // channel of the row
            float cA = 1.f, cK = 0.f, cV = 0.f;
#pragma unroll
            for (int wp = 0; wp < C::PW; ++wp) {
                const float a = sw[(wp * 3 + 0) * SC + ch];
                cK = fmaf(a, cK, sw[(wp * 3 + 1) * SC + ch]);
                cV = fmaf(a, cV, sw[(wp * 3 + 2) * SC + ch]);
                cA *= a;
            }
            if (c > 0 && publish) {
                uint64_t *agg = p.agg + chunk_id * 3 * SC;
                st_relaxed_gpu_u64(agg + ch, tagged(tag, cA));
                st_relaxed_gpu_u64(agg + SC + ch, tagged(tag, cK));
                st_relaxed_gpu_u64(agg + 2 * SC + ch, tagged(tag, cV));
            }
            float Hk = 0.f, Hv = 0.f;
            if (c == 0) {
                if (p.h0k) Hk = p.h0k[(size_t)bh * C::DH + gch];
                if (p.h0v) Hv = p.h0v[(size_t)bh * C::DH + gch];
            } else {
                // the same walk as the full-row scan: LBW predecessors per round, an inclusive
                // state ends it, an aggregate is composed in, a missing record ends the round
                float xA = 1.f, xK = 0.f, xV = 0.f;
                const uint64_t t_start = globaltimer_ns();
                uint32_t spins = 0;
                int j = c - 1;
                for (bool first = true;; first = false) {
                    if (!first) read_window(item, j, ch, w);
                    bool done = false, stop = false;
                    int passed = 0;
#pragma unroll
                    for (int u = 0; u < C::LBW; ++u) {
                        if (done || stop || j - u < 0) continue;
                        auto ok = [&](int e) { return (uint32_t)(w[u][e] >> 32) == tag; };
                        auto val = [&](int e) { return __uint_as_float((uint32_t)w[u][e]); };
                        if (ok(0) && ok(1)) {
                            Hk = fmaf(xA, val(0), xK);
                            Hv = fmaf(xA, val(1), xV);
                            done = true;
                        } else if (ok(2) && ok(3) && ok(4)) {
                            xK = fmaf(xA, val(3), xK);
                            xV = fmaf(xA, val(4), xV);
                            xA *= val(2);
                            ++passed;
                        } else {
                            stop = true;
                        }
                    }
                    if (done) break;
                    j -= passed;
                    if (passed == 0) {
                        if ((++spins & 7u) == 0u && globaltimer_ns() - t_start > p.wait_ns) {
                            record_error(hdr, RAT_ERR_TIMEOUT, 0x200u);
                            break;
                        }
                        __nanosleep(32);
                    }
                }
            }
            const float outK = fmaf(cA, Hk, cK), outV = fmaf(cA, Hv, cV);
            if (publish) {
                uint64_t *pre = p.pre + chunk_id * 2 * SC;
                st_relaxed_gpu_u64(pre + ch, tagged(tag, outK));
                st_relaxed_gpu_u64(pre + SC + ch, tagged(tag, outV));
            }
            if (c == p.nchunks - 1) {
                if (p.hTk) p.hTk[(size_t)bh * C::DH + gch] = outK;
                if (p.hTv) p.hTv[(size_t)bh * C::DH + gch] = outV;
            }
            float hK = Hk, hV = Hv;
#pragma unroll
            for (int wp = 0; wp < C::PW; ++wp) {
                const float a = sw[(wp * 3 + 0) * SC + ch];
                const float bk = sw[(wp * 3 + 1) * SC + ch];
                const float bv = sw[(wp * 3 + 2) * SC + ch];
                sw[(wp * 3 + 0) * SC + ch] = hK;
                sw[(wp * 3 + 1) * SC + ch] = hV;
                hK = fmaf(a, hK, bk);
                hV = fmaf(a, hV, bv);
            }
        }
        pipe_sync();

        // ---- pass 2: rerun the segment from its carry with the kept gates; write k~ (rotated)
        // and v~
        f2_t hk[NP], hv[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            const float2 *s2 = reinterpret_cast<const float2 *>(sw) + cl + 16 * q;
            const float2 ck = s2[((pwarp * 3 + 0) * SC) / 2];
            const float2 cv = s2[((pwarp * 3 + 1) * SC) / 2];
            hk[q] = f2_fma(eA[q], f2(ck.x, ck.y), eK[q]);
            hv[q] = f2_fma(eA[q], f2(cv.x, cv.y), eV[q]);
        }
        // RoPE: frequencies 32 slice + 2 cl (+1) at the segment's first row, advanced one
        // position per row; pair 0 (first half) takes x cos - x' sin, pair 1 x' cos + x sin
        f2_t rc = kOne2, rs = kZero2, sc = kOne2, ss = kZero2, nss = kZero2;
        if (p.rope) {
            const long long pos = p.pos0 + t0 + seg * R;
            float c2[2], s2v[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int f = 32 * slice + 2 * cl + u;
                if (p.rope_f32) rope_cs_f32((int)pos, s_theta_f[f], c2[u], s2v[u]);
                else rope_cs(pos, s_theta[f], c2[u], s2v[u]);
            }
            rc = f2(c2[0], c2[1]);
            rs = f2(s2v[0], s2v[1]);
            const int f0 = 32 * slice + 2 * cl;
            sc = f2(s_step_c[f0], s_step_c[f0 + 1]);
            ss = f2(s_step_s[f0], s_step_s[f0 + 1]);
            nss = f2(-s_step_s[f0], -s_step_s[f0 + 1]);
        }
        const f2_t kNegOne2 = f2(-1.f, -1.f);
        uint8_t *yk = static_cast<uint8_t *>(p.yk) + 64 * slice;
        uint8_t *yv = static_cast<uint8_t *>(p.yv) + 64 * slice;
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = seg * R + i;
            const int off = soff(r < rows ? r : rows - 1) - 4 * cl;
            f2_t xk[NP], xv[NP];
            Lane<__nv_bfloat16>::template load<128>(sk + off, cl, xk);
            Lane<__nv_bfloat16>::template load<128>(sv + off, cl, xv);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const f2_t og = gate_complement2(G[i][q]);
                hk[q] = f2_fma(G[i][q], hk[q], f2_mul(og, xk[q]));
                hv[q] = f2_fma(G[i][q], hv[q], f2_mul(og, xv[q]));
            }
            f2_t ok[NP] = {hk[0], hk[1]};
            if (p.rope) {
                const f2_t nrs = f2_mul(rs, kNegOne2);
                ok[0] = f2_fma(hk[1], nrs, f2_mul(hk[0], rc));
                ok[1] = f2_fma(hk[0], rs, f2_mul(hk[1], rc));
                const f2_t nc = f2_fma(rc, sc, f2_mul(rs, nss));
                rs = f2_fma(rs, sc, f2_mul(rc, ss));
                rc = nc;
            }
            if (r < rows) {
                const size_t go = (row0 + r) * (C::DH * 2);
                Lane<__nv_bfloat16>::template store<128>(yk + go, cl, ok);
                Lane<__nv_bfloat16>::template store<128>(yv + go, cl, hv);
            }
        }
        pipe_sync();
    }
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
    return 16384 / (d * eb);               // one 16 KiB tile per tensor
}

size_t recur_workspace_bytes(int BH, int T, int d, int dtype) {
    const size_t tc = (size_t)recur_chunk_rows(d, dtype);
    const size_t nch = (size_t)BH * ((T + tc - 1) / tc);
    return sizeof(WsHeader) + align256(nch * 3 * d * 8) + align256(nch * 2 * d * 8);
}

template <typename E, int DH>
static int launch_one(const RecurParams &p, void *stream) {
    using C = ScanCfg<E, DH>;
    auto kern = p.reset > 0 ? recur_kernel<E, DH, true> : recur_kernel<E, DH, false>;
    static std::atomic<uint64_t> attr_done[2] = {{0}, {0}};
    const int st = set_smem_attr(reinterpret_cast<const void *>(kern), C::SMEM, &attr_done[p.reset > 0]);
    if (st != RAT_OK) return st;
    const int sms = current_sm_count();
    if (sms <= 0) return RAT_ERR_CUDA;
    // persistent: one CTA per SM, each walking chunks in ticket order
    const long long total = (long long)p.BH * p.nchunks;
    const unsigned grid = (unsigned)(total < sms ? total : sms);
    kern<<<grid, C::THREADS, C::SMEM, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

static PFN_cuTensorMapEncodeTiled_v12000 scan_encode_fn() {
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

// 5-D view of a (rows, 128) bf16 tensor, rows a multiple of 16: channel x < 64 of a half,
// segment-in-warp u < 2 (8 rows apart), half y < 2 (64 channels apart), row-in-segment i < 8,
// 16-row group g; box (32, 2, 2, 8, 8) = one 128-row chunk of one slice.
static bool slice_map(CUtensorMap *m, const void *base, uint64_t rows) {
    auto fn = scan_encode_fn();
    if (!fn) return false;
    constexpr uint64_t row = 128 * 2;
    cuuint64_t dims[5] = {64, 2, 2, 8, rows / 16};
    cuuint64_t strides[4] = {8 * row, 64 * 2, row, 16 * row};
    cuuint32_t box[5] = {32, 2, 2, 8, (cuuint32_t)SliceCfg::TC / 16};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The channel-sliced scan; returns RAT_ERR_UNSUPPORTED when the tensor maps cannot be built
// (the caller then runs the full-row scan).
static int launch_slice(const RecurParams &p, void *stream) {
    using C = SliceCfg;
    SliceParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.r = p;
    sp.r.nchunks = (p.T + C::TC - 1) / C::TC;
    const uint64_t rows = (uint64_t)p.BH * (uint64_t)p.T;
    if (!slice_map(&sp.tm_a, p.a, rows) || !slice_map(&sp.tm_k, p.k, rows) || !slice_map(&sp.tm_v, p.v, rows))
        return RAT_ERR_UNSUPPORTED;
    static std::atomic<uint64_t> attr_done{0};
    const int st = set_smem_attr(reinterpret_cast<const void *>(recur_slice_kernel), C::SMEM, &attr_done);
    if (st != RAT_OK) return st;
    const int sms = current_sm_count();
    if (sms <= 0) return RAT_ERR_CUDA;
    const long long total = 2ll * p.BH * sp.r.nchunks;
    const unsigned grid = (unsigned)(total < sms ? total : sms);
    recur_slice_kernel<<<grid, C::THREADS, C::SMEM, static_cast<cudaStream_t>(stream)>>>(sp);
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

int launch_recur(const RecurParams &p, int dtype, void *stream) {
    // bf16, d 128, full sequence, T a multiple of 16: the channel-sliced scan
    if (dtype == RAT_BF16 && p.d == 128 && p.reset == 0 && p.T % 16 == 0) {
        const int st = launch_slice(p, stream);
        if (st != RAT_ERR_UNSUPPORTED) return st;
    }
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
