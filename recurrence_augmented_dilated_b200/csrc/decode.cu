// decode.cu -- one new token per sequence against the D-fold compressed KV cache.
//
// RAT+ abstract (dilated attention with an optional local window; D-fold smaller KV cache) and
// "RAT+ Deep Dive" section 2.1 (the recurrence state carries what dilation skips).  For the token
// at position t of slice (b, h):
//   1. state update  h_k = g h_k + (1-g) k,  h_v = g h_v + (1-g) v   (float32, g = sigmoid(a));
//      k~_t = RoPE(h_k, t), v~_t = h_v, both rounded to the cache dtype; with the chunk-local
//      recurrence of RAT (abstract of "RAT: Bridging RNN Efficiency and Attention Accuracy"),
//      h is dropped first when t is a multiple of the block length L;
//   2. append k~_t, v~_t to dil entry (t - D + 1) / D if t mod D = D - 1, and to ring slot t mod W;
//   3. attention of q^ = RoPE(q, t) over the prefill key set S(t): dil entries whose position
//      i*D + D - 1 <= t - We, ring positions t - We < j < t, and the token itself.
// Memory-bound: every key is one 16-byte load per lane for K and one for V.  The keys of a
// slice are split over `splits` CTAs; each CTA keeps an online softmax per 16-lane group,
// merges its groups and warps, and writes (max, sum, o) to the workspace; the last CTA of the
// slice (atomic ticket, no waiting) merges the splits by log-sum-exp and resets the ticket.
// Split 0 alone does steps 1-2 and adds the token itself to its softmax.  With the fixed-window
// recurrence ("RAT+ Deep Dive" section 2.1, L* = 64) step 1 reruns the recurrence from zero over
// the raw rows of the 63 positions before t (a raw ring in the cache) instead of reading a
// carried state, and the token's raw rows take the ring slot of position t - 64; that pass loads
// two rows at a time so the form keeps the uniform form's registers and CTAs per SM.
// No CTA reads what another writes in the same launch: the new dil entry (position t) is never
// older than the window, and the ring slot written held position t - W, outside the window.
#include <mutex>

#include "common.cuh"

namespace rat {

namespace {
constexpr int kThreads = 128;       // 4 warps; 16 lanes x 8 channels = one d=128 bf16 row
constexpr int kWarps = kThreads / 32;

RAT_DEVICE void load8(const void *p, float *x) {      // 8 bf16 -> float
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z); x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
}
RAT_DEVICE void unpack8(uint4 u, float *x) {          // 8 bf16 -> float
    x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z); x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
}
RAT_DEVICE uint4 pack8(const float *x) {
    return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                      pack_bf16(x[6], x[7]));
}
}  // namespace

// Template on d: 16 lanes per row for d = 128 (8 bf16 each), 8 lanes for d = 64.  PAGED: the
// dilated entries live in pages of a pool found through a page table, and every sequence has
// its own position (read from seq_pos, advanced by the last CTA of the sequence).
// SINKS: the first n_sink positions are kept in sink rows and join every key set.
// WINDOW: the fixed-window recurrence (raw rings; p.window_rec > 0).  Its split 0 also reruns
// the recurrence over the raw ring, a few rows at a time.  Every instantiation is held to the
// CTAs per SM of the uniform form (five; six for the paged form).
template <int DH, bool PAGED, bool SINKS, bool WINDOW>
__global__ void __launch_bounds__(kThreads, PAGED ? 6 : 5) decode_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int LPR = DH / 8;                 // lanes per key row
    constexpr int GPW = 32 / LPR;               // key groups per warp
    constexpr int RB = DH * 2;                  // row bytes (bf16)
    const int split = blockIdx.x, bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = lane / LPR, cl = lane % LPR;   // key group inside the warp, lane inside row
    const long long t = PAGED ? p.seq_pos[b] : p.t;
    const long long D = p.Dh[h];
    const long long We = p.W > 1 ? p.W : 1;
    const long long cap = PAGED ? (long long)p.max_pages << p.page_shift : p.Tcap / D;
    // pool row of dil entry idx of this slice; a page index outside the pool marks the entry
    // missing (and records the error) instead of reading outside the pool
    const int32_t *ptab = PAGED ? p.page_table + (size_t)bh * p.max_pages : nullptr;
    auto dil_row = [&](long long idx, bool &ok) -> size_t {
        if (!PAGED) {
            ok = true;
            return (size_t)b * p.total_cap + p.off[h] + idx;
        }
        const int32_t pg = __ldg(ptab + (idx >> p.page_shift));
        ok = (uint32_t)pg < (uint32_t)p.n_pages;
        if (!ok) record_error(p.hdr, RAT_ERR_INVALID, 0x400u);
        return ((size_t)(ok ? pg : 0) << p.page_shift) + (size_t)(idx & ((1ll << p.page_shift) - 1));
    };
    const bool first_half = cl < LPR / 2;

    // the new token's query, rotated; every lane group holds a copy of its 8 channels
    float q[8];
    load8(static_cast<const uint8_t *>(p.q) + (size_t)bh * RB + cl * 16, q);
    if (p.rope) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float cs, sn;
            rope_cs(t, p.theta[(cl * 8 + j) % (DH / 2)], cs, sn);
            const float partner = __shfl_xor_sync(0xffffffffu, q[j], LPR / 2);
            q[j] = first_half ? q[j] * cs - partner * sn : q[j] * cs + partner * sn;
        }
    }

    // key list of this slice: [0, n_dil) dil entries, then [n_dil, n_dil + n_ring) ring
    // positions, then (SINKS) the sinks older than the window that are not chunk ends (sink s is
    // position s + s / (D-1))
    long long n_dil = (t - We + 1) >= D ? (t - We + 1) / D : 0;
    if (n_dil > cap) n_dil = cap;
    const long long r_lo = max(0ll, t - We + 1);           // first ring position in the window
    const long long n_ring = t - r_lo;                      // positions r_lo .. t-1
    long long n_snk = 0;
    if constexpr (SINKS) {
        const long long s_lim = min((long long)p.n_sink, r_lo);
        n_snk = D > 1 ? s_lim - s_lim / D : 0;
    }
    const long long n_keys = n_dil + n_ring + n_snk;
    const long long k_lo = n_keys * split / p.splits, k_hi = n_keys * (split + 1) / p.splits;

    // paged: the pools; otherwise this slice's first entry
    const size_t dil0 = PAGED ? 0 : ((size_t)b * p.total_cap + p.off[h]) * RB;
    const uint8_t *kdil = static_cast<const uint8_t *>(p.kdil) + dil0;
    const uint8_t *vdil = static_cast<const uint8_t *>(p.vdil) + dil0;
    const uint8_t *kwin = p.kwin ? static_cast<const uint8_t *>(p.kwin) + (size_t)bh * p.W * RB : nullptr;
    const uint8_t *vwin = p.vwin ? static_cast<const uint8_t *>(p.vwin) + (size_t)bh * p.W * RB : nullptr;

    float m = -INFINITY, l = 0.f, o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = 0.f;

    // fixed-window form, split 0: the affine map of the raw rows max(0, t - Lw + 1) .. t - 1 (the
    // recurrence from zero over them), composed in kWarps * GPW segments, one per lane group with
    // kBatch rows' loads in flight at a time; warp 0 folds the segments in order below
    constexpr int kSegs = kWarps * (32 / (DH / 8));
    __shared__ float s_wa[WINDOW ? kSegs : 1][DH], s_wk[WINDOW ? kSegs : 1][DH], s_wv[WINDOW ? kSegs : 1][DH];
    if (WINDOW && split == 0) {
        const int seg = warp * GPW + grp;
        const long long lo = max(0ll, t - p.window_rec + 1), n = t - lo;
        const long long r0 = lo + n * seg / kSegs, r1 = lo + n * (seg + 1) / kSegs;
        constexpr int kMaxSeg = (kWindowRows + kSegs - 1) / kSegs;      // rows per segment
        constexpr int kBatch = 2;            // rows whose loads are in flight together (registers)
        const size_t ring = (size_t)bh * p.window_rec;
        float A[8], K[8], V[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) { A[j] = 1.f; K[j] = 0.f; V[j] = 0.f; }
#pragma unroll
        for (int i0 = 0; i0 < kMaxSeg; i0 += kBatch) {
            uint4 ra[kBatch], rk[kBatch], rv[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                if (r0 + i0 + i < r1) {
                    const size_t off = (ring + (size_t)((r0 + i0 + i) % p.window_rec)) * RB + cl * 16;
                    ra[i] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.araw) + off));
                    rk[i] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.kraw) + off));
                    rv[i] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.vraw) + off));
                }
            }
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                if (r0 + i0 + i < r1) {
                    float fa[8], fk[8], fv[8];
                    unpack8(ra[i], fa);
                    unpack8(rk[i], fk);
                    unpack8(rv[i], fv);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float g, omg;
                        forget_gate(fa[j], g, omg);
                        K[j] = fmaf(g, K[j], omg * fk[j]);
                        V[j] = fmaf(g, V[j], omg * fv[j]);
                        A[j] *= g;
                    }
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {      // both lanes of a pair hold the same group values
            s_wa[seg][cl * 8 + j] = A[j];
            s_wk[seg][cl * 8 + j] = K[j];
            s_wv[seg][cl * 8 + j] = V[j];
        }
        __syncthreads();                   // split is uniform over the CTA
    }

    // keys of this split: lane set s = warp*GPW + grp takes keys k_lo + s + m*kLanesets, KPI at a
    // time (their K and V rows in flight together, kept as packed bf16).  The loop runs on the
    // warp's first key so every lane of a warp iterates the same number of times (the
    // dot-product shuffles below need all 32 lanes).
    constexpr int kLanesets = kWarps * GPW;
    constexpr int KPI = 4;
    const int set = warp * GPW + grp;
    for (long long base = k_lo + warp * GPW; base < k_hi; base += KPI * kLanesets) {
        uint4 kr[KPI], vr[KPI];
        bool have[KPI];
#pragma unroll
        for (int u = 0; u < KPI; ++u) {
            const long long idx = base + grp + (long long)u * kLanesets;
            have[u] = idx < k_hi;
            // lanes of a warp may disagree on `have`; loads are predicated, shuffles are not
            if (have[u]) {
                const uint8_t *kp, *vp;
                if (idx < n_dil) {
                    if constexpr (PAGED) {
                        bool ok;
                        const size_t row = dil_row(idx, ok);
                        have[u] = ok;
                        kp = kdil + row * RB;
                        vp = vdil + row * RB;
                    } else {
                        kp = kdil + (size_t)idx * RB;
                        vp = vdil + (size_t)idx * RB;
                    }
                } else if (!SINKS || idx < n_dil + n_ring) {
                    const long long pos = r_lo + (idx - n_dil);
                    kp = kwin + (size_t)(pos % p.W) * RB;
                    vp = vwin + (size_t)(pos % p.W) * RB;
                } else {
                    const long long s = idx - n_dil - n_ring;
                    const size_t row = (size_t)bh * p.n_sink + (size_t)(s + s / (D - 1));
                    kp = static_cast<const uint8_t *>(p.ksink) + row * RB;
                    vp = static_cast<const uint8_t *>(p.vsink) + row * RB;
                }
                kr[u] = __ldg(reinterpret_cast<const uint4 *>(kp + cl * 16));
                vr[u] = __ldg(reinterpret_cast<const uint4 *>(vp + cl * 16));
            } else {
                kr[u] = make_uint4(0u, 0u, 0u, 0u);
                vr[u] = kr[u];
            }
            if (PAGED && !have[u]) {            // an entry without a page
                kr[u] = make_uint4(0u, 0u, 0u, 0u);
                vr[u] = kr[u];
            }
        }
        float sc[KPI];
#pragma unroll
        for (int u = 0; u < KPI; ++u) {
            const uint32_t ku[4] = {kr[u].x, kr[u].y, kr[u].z, kr[u].w};
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                dot = fmaf(q[2 * i], bf16_lo(ku[i]), dot);
                dot = fmaf(q[2 * i + 1], bf16_hi(ku[i]), dot);
            }
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            sc[u] = have[u] ? dot * p.scale_log2 : -INFINITY;
        }
        // one rescale for the KPI keys
        const float mb = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
        const float mn = fmaxf(m, mb);
        if (mn != -INFINITY) {
            const float corr = ex2_approx(m - mn);        // m = -inf -> 0
            l *= corr;
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] *= corr;
#pragma unroll
            for (int u = 0; u < KPI; ++u) {
                const float pj = ex2_approx(sc[u] - mn);   // masked keys: -inf -> 0
                l += pj;
                const uint32_t vu[4] = {vr[u].x, vr[u].y, vr[u].z, vr[u].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    o[2 * i] = fmaf(pj, bf16_lo(vu[i]), o[2 * i]);
                    o[2 * i + 1] = fmaf(pj, bf16_hi(vu[i]), o[2 * i + 1]);
                }
            }
            m = mn;
        }
    }

    // split 0: recurrence update, cache append, and the token itself as a key (group 0 of warp 0)
    if (split == 0 && warp == 0) {
        const uint4 ku = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.k) + (size_t)bh * RB + cl * 16));
        const uint4 vu = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.v) + (size_t)bh * RB + cl * 16));
        const uint4 au = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.a) + (size_t)bh * RB + cl * 16));
        float kn[8], vn[8], an[8];
        unpack8(ku, kn);
        unpack8(vu, vn);
        unpack8(au, an);
        float *hk = p.hk + (size_t)bh * DH + cl * 8;
        float *hv = p.hv + (size_t)bh * DH + cl * 8;
        // the state entering position t: the cache's (0 before a block start of the chunk-local
        // recurrence), or, for the fixed-window form, the recurrence rerun from zero over the raw
        // rows of positions max(0, t - Lw + 1) .. t - 1
        float hsk[8], hsv[8];
        if constexpr (WINDOW) {
#pragma unroll
            for (int j = 0; j < 8; ++j) { hsk[j] = 0.f; hsv[j] = 0.f; }
            for (int sg = 0; sg < kSegs; ++sg) {       // the segments' maps, oldest first
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int c = cl * 8 + j;
                    hsk[j] = fmaf(s_wa[sg][c], hsk[j], s_wk[sg][c]);
                    hsv[j] = fmaf(s_wa[sg][c], hsv[j], s_wv[sg][c]);
                }
            }
        } else {
            const bool fresh = p.reset > 0 && t % p.reset == 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                hsk[j] = fresh ? 0.f : hk[j];
                hsv[j] = fresh ? 0.f : hv[j];
            }
        }
        float sk[8], sv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float g, omg;
            forget_gate(an[j], g, omg);
            sk[j] = fmaf(g, hsk[j], omg * kn[j]);
            sv[j] = fmaf(g, hsv[j], omg * vn[j]);
        }
        float kt[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) kt[j] = sk[j];
        if (p.rope) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float cs, sn;
                rope_cs(t, p.theta[(cl * 8 + j) % (DH / 2)], cs, sn);
                const float partner = __shfl_xor_sync(0xffffffffu, sk[j], LPR / 2);
                kt[j] = first_half ? sk[j] * cs - partner * sn : sk[j] * cs + partner * sn;
            }
        }
        const uint4 kpk = pack8(kt), vpk = pack8(sv);
        if (grp == 0) {
#pragma unroll
            for (int j = 0; j < 8; ++j) { hk[j] = sk[j]; hv[j] = sv[j]; }
            if (t % D == D - 1) {
                bool ok = t / D < cap;
                if (ok) {
                    const size_t row = dil_row(t / D, ok);
                    if (ok) {
                        uint8_t *kd = static_cast<uint8_t *>(p.kdil) + row * RB;
                        uint8_t *vd = static_cast<uint8_t *>(p.vdil) + row * RB;
                        *reinterpret_cast<uint4 *>(kd + cl * 16) = kpk;
                        *reinterpret_cast<uint4 *>(vd + cl * 16) = vpk;
                    }
                } else if (PAGED) {
                    record_error(p.hdr, RAT_ERR_INVALID, 0x401u);     // no page for the entry
                }
            }
            if (SINKS && t < p.n_sink) {
                uint8_t *ks = static_cast<uint8_t *>(p.ksink) + ((size_t)bh * p.n_sink + (size_t)t) * RB;
                uint8_t *vs = static_cast<uint8_t *>(p.vsink) + ((size_t)bh * p.n_sink + (size_t)t) * RB;
                *reinterpret_cast<uint4 *>(ks + cl * 16) = kpk;
                *reinterpret_cast<uint4 *>(vs + cl * 16) = vpk;
            }
            if (WINDOW) {                    // the token's raw rows: slot t mod Lw held t - Lw
                const size_t off = ((size_t)bh * p.window_rec + (size_t)(t % p.window_rec)) * RB + cl * 16;
                *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(p.kraw) + off) = ku;
                *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(p.vraw) + off) = vu;
                *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(p.araw) + off) = au;
            }
            if (p.W > 0) {
                uint8_t *kw = static_cast<uint8_t *>(p.kwin) + ((size_t)bh * p.W + (size_t)(t % p.W)) * RB;
                uint8_t *vw = static_cast<uint8_t *>(p.vwin) + ((size_t)bh * p.W + (size_t)(t % p.W)) * RB;
                *reinterpret_cast<uint4 *>(kw + cl * 16) = kpk;
                *reinterpret_cast<uint4 *>(vw + cl * 16) = vpk;
            }
        }
        // the token itself, as stored in the cache (rounded), attended by lane group 0
        float kr[8], vr[8];
        kr[0] = bf16_lo(kpk.x); kr[1] = bf16_hi(kpk.x); kr[2] = bf16_lo(kpk.y); kr[3] = bf16_hi(kpk.y);
        kr[4] = bf16_lo(kpk.z); kr[5] = bf16_hi(kpk.z); kr[6] = bf16_lo(kpk.w); kr[7] = bf16_hi(kpk.w);
        vr[0] = bf16_lo(vpk.x); vr[1] = bf16_hi(vpk.x); vr[2] = bf16_lo(vpk.y); vr[3] = bf16_hi(vpk.y);
        vr[4] = bf16_lo(vpk.z); vr[5] = bf16_hi(vpk.z); vr[6] = bf16_lo(vpk.w); vr[7] = bf16_hi(vpk.w);
        float dot = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) dot = fmaf(q[j], kr[j], dot);
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        if (grp == 0) {
            const float s = dot * p.scale_log2;
            const float mn = fmaxf(m, s);
            const float corr = exp2f(m - mn), pj = exp2f(s - mn);
            l = fmaf(l, corr, pj);
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] = fmaf(o[j], corr, pj * vr[j]);
            m = mn;
        }
    }

    // merge the lane groups of each warp, then the warps, through shared memory
    __shared__ float s_m[kWarps * 4], s_l[kWarps * 4];
    __shared__ float s_o[kWarps * 4][DH];
    s_m[set] = m;            // every lane of the group writes the same value
    s_l[set] = l;
#pragma unroll
    for (int j = 0; j < 8; ++j) s_o[set][cl * 8 + j] = o[j];
    __syncthreads();
    // CTA merge: thread c < DH owns channel c
    if (tid < DH) {
        float M = -INFINITY;
        for (int s2 = 0; s2 < kLanesets; ++s2) M = fmaxf(M, s_m[s2]);
        float L = 0.f, O = 0.f;
        for (int s2 = 0; s2 < kLanesets; ++s2) {
            const float w = s_m[s2] == -INFINITY ? 0.f : exp2f(s_m[s2] - M);
            L = fmaf(s_l[s2], w, L);
            O = fmaf(s_o[s2][tid], w, O);
        }
        p.part_o[((size_t)bh * p.splits + split) * DH + tid] = O;
        if (tid == 0) {
            p.part_ml[((size_t)bh * p.splits + split) * 2 + 0] = M;
            p.part_ml[((size_t)bh * p.splits + split) * 2 + 1] = L;
        }
        __threadfence();
    }
    __shared__ uint32_t s_last;
    __syncthreads();
    if (tid == 0) {
        s_last = atomicAdd(&p.tickets[bh], 1u) == (uint32_t)p.splits - 1;
        if (PAGED) {
            // every CTA of the sequence has read its position (at its start): the last one to
            // finish advances it for the next step and rearms the ticket
            const uint32_t n = (uint32_t)(p.H * p.splits);
            if (atomicAdd(&p.seq_ticket[b], 1u) == n - 1) {
                p.seq_ticket[b] = 0u;
                p.seq_pos[b] = t + 1;
            }
        }
    }
    __syncthreads();
    if (!s_last) return;
    // last CTA of the slice: merge the splits
    if (tid < DH) {
        float M = -INFINITY;
        for (int s2 = 0; s2 < p.splits; ++s2) M = fmaxf(M, __ldcg(&p.part_ml[((size_t)bh * p.splits + s2) * 2]));
        float L = 0.f, O = 0.f;
        for (int s2 = 0; s2 < p.splits; ++s2) {
            const float ms = __ldcg(&p.part_ml[((size_t)bh * p.splits + s2) * 2]);
            const float w = ms == -INFINITY ? 0.f : exp2f(ms - M);
            L = fmaf(__ldcg(&p.part_ml[((size_t)bh * p.splits + s2) * 2 + 1]), w, L);
            O = fmaf(__ldcg(&p.part_o[((size_t)bh * p.splits + s2) * DH + tid]), w, O);
        }
        const float r = O / L;
        __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(p.o) + (size_t)bh * DH + tid;
        *out = __float2bfloat16_rn(r);
    }
    if (tid == 0) p.tickets[bh] = 0u;
}

int decode_splits(int B, int H, int Tcap, const int32_t *Dh, int W) {
    long long max_keys = 0;
    for (int h = 0; h < H; ++h) {
        const long long k = Tcap / Dh[h] + W;
        max_keys = k > max_keys ? k : max_keys;
    }
    return decode_splits_for_keys(B, H, max_keys);
}

int decode_splits_for_keys(int B, int H, long long max_keys) {
    // aim for about 12 CTAs per SM over the 148 SMs, and at least ~64 keys per split (measured on
    // the 32 x 32-slice, 1151-key workload: 2 splits per slice beat 1, 3, 4, 5 and 7)
    const long long bh = (long long)B * H;
    long long s = (148ll * 12 + bh - 1) / bh;
    const long long by_keys = (max_keys + 63) / 64;
    if (s > by_keys) s = by_keys;
    if (s < 1) s = 1;
    if (s > 64) s = 64;
    return (int)s;
}

// header, per-slice tickets, per-split (max, sum) and o partials, per-sequence tickets
size_t decode_workspace_bytes(int B, int H, int d, int splits) {
    const size_t bh = (size_t)B * H;
    return sizeof(WsHeader) + align256(bh * 4) + align256(bh * splits * 2 * 4) +
           align256(bh * splits * d * 4) + align256((size_t)B * 4);
}

int launch_decode(const DecodeParams &p, int dtype, void *stream, bool paged) {
    if (dtype != RAT_BF16) return RAT_ERR_UNSUPPORTED;
    dim3 grid((unsigned)p.splits, (unsigned)(p.B * p.H));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool sinks = p.n_sink > 0;
    if (paged && sinks) return RAT_ERR_UNSUPPORTED;
    const bool window = p.window_rec > 0;
    if (paged && window) return RAT_ERR_UNSUPPORTED;
    if (p.d == 128) {
        if (paged) decode_kernel<128, true, false, false><<<grid, kThreads, 0, s>>>(p);
        else if (window && sinks) decode_kernel<128, false, true, true><<<grid, kThreads, 0, s>>>(p);
        else if (window) decode_kernel<128, false, false, true><<<grid, kThreads, 0, s>>>(p);
        else if (sinks) decode_kernel<128, false, true, false><<<grid, kThreads, 0, s>>>(p);
        else decode_kernel<128, false, false, false><<<grid, kThreads, 0, s>>>(p);
    } else if (p.d == 64) {
        if (paged) decode_kernel<64, true, false, false><<<grid, kThreads, 0, s>>>(p);
        else if (window && sinks) decode_kernel<64, false, true, true><<<grid, kThreads, 0, s>>>(p);
        else if (window) decode_kernel<64, false, false, true><<<grid, kThreads, 0, s>>>(p);
        else if (sinks) decode_kernel<64, false, true, false><<<grid, kThreads, 0, s>>>(p);
        else decode_kernel<64, false, false, false><<<grid, kThreads, 0, s>>>(p);
    } else {
        return RAT_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

}  // namespace rat

// ------------------------------------------------------------------------------ no-allocation entry
// A decode call needs a small scratch area (per-split partial results and per-slice tickets).
// Some callers cannot hand the library a device buffer for it: their device memory is owned by a
// host framework or planned up front as a fixed arena, and they have no way to obtain an extra
// allocation.  rat_dilated_decode_noalloc serves them from this fixed array in the library's own
// device image (every GPU that loads the library holds it until the process exits).
namespace rat {
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;     // 8 MiB
constexpr int kNoAllocMaxDevices = 64;
}  // namespace

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_scratch_mutex;
void *g_scratch_addr[kNoAllocMaxDevices];   // device address of g_decode_scratch, per device
}  // namespace

}  // namespace rat

extern "C" int rat_dilated_decode_noalloc(const void *q, const void *k, const void *v,
                                          const void *gate_logit, rat_kv_cache *cache, void *o,
                                          float rope_base, float scale, void *stream) {
    using namespace rat;
    const size_t need = rat_decode_workspace_bytes(cache);
    if (need == 0) return RAT_ERR_INVALID;                  // invalid cache description
    if (need > kNoAllocScratchBytes) return RAT_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RAT_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return RAT_ERR_UNSUPPORTED;
    void *ptr = nullptr;
    {
        // first call on this device: look up the array's device address (host code cannot use
        // the symbol itself as a device pointer)
        std::lock_guard<std::mutex> lock(g_scratch_mutex);
        if (!g_scratch_addr[dev]) {
            void *a = nullptr;
            if (cudaGetSymbolAddress(&a, g_decode_scratch) != cudaSuccess || !a) return RAT_ERR_CUDA;
            g_scratch_addr[dev] = a;
        }
        ptr = g_scratch_addr[dev];
    }
    // the array keeps the previous call's contents: the header (error word) and the per-slice
    // tickets must start at zero
    const size_t bh = (size_t)cache->B * cache->H;
    if (cudaMemsetAsync(ptr, 0, sizeof(WsHeader) + align256(bh * 4), static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return RAT_ERR_CUDA;
    return rat_dilated_decode(q, k, v, gate_logit, cache, o, rope_base, scale, ptr, kNoAllocScratchBytes, stream);
}

