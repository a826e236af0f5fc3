// compress.cu -- build / extend the D-fold compressed KV cache from recurrence outputs.
//
// RAT+ abstract: dilation keeps every D-th key, which cuts the KV cache D-fold; the local
// window keeps the W most recent positions.  For the T new positions pos0 .. pos0+T-1 of every
// (b, h) this kernel copies
//   - each chunk end p = i*D_h + D_h - 1 (i < cap_h) to dil entry i of head h, and
//   - each of the last min(W, T) positions p to ring slot p mod W,
//   - each position p < n_sink to sink row p (attention sinks),
// for k~ and v~, bit for bit; and copies the final recurrence state into the cache.
// One CTA per (row block, b*h); 16-byte vector copies, one row per LPR lanes, four rows per
// thread in flight at once.  The paged form (one sequence per call) writes the dil entries into
// the pool rows the page table names, and sets the sequence's position.
#include <algorithm>

#include "common.cuh"

namespace rat {

// PAGED: the paged form (one sequence per call, dil entries through the page table)
template <bool PAGED>
__global__ void __launch_bounds__(256) compress_kernel(const __grid_constant__ CompressParams p) {
    // flat grid: per batch row, head h owns CTAs blk0[h] .. blk0[h+1]-1
    const int per_b = p.blk0[p.H];
    const int b = (int)blockIdx.x / per_b, rb = (int)blockIdx.x % per_b;
    int h = 0;
    while (rb >= p.blk0[h + 1]) ++h;
    const int bh = b * p.H + h;                                  // input slice
    constexpr bool paged = PAGED;
    const int bhc = paged ? p.seq * p.H + h : bh;                // cache slice
    const int blk = rb - p.blk0[h], nblk = p.blk0[h + 1] - p.blk0[h];
    const long long D = p.Dh[h];
    const long long cap = paged ? (long long)p.max_pages << p.page_shift : p.Tcap / D;
    const long long end = p.pos0 + p.T;
    const long long i_lo = p.pos0 / D;                       // first chunk end >= pos0
    const long long i_hi = min(end / D, cap);                // chunk ends < end, within capacity
    const long long n_dil = max(0ll, i_hi - i_lo);
    const long long r_lo = max(p.pos0, end - (long long)p.W);  // ring positions [r_lo, end)
    const long long n_ring = p.W > 0 ? end - r_lo : 0;
    const long long n_sk = max(0ll, min(end, (long long)p.n_sink) - p.pos0);   // sink rows
    const int row_bytes = p.d * p.esize;
    const int lpr = row_bytes / 16;                          // lanes per row
    const int rows_per_pass = blockDim.x / lpr;
    const int lane_r = threadIdx.x / lpr, lane_c = threadIdx.x % lpr;
    const long long per = n_dil + n_ring + n_sk;            // rows of one tensor
    const long long njobs = 2 * per;                          // (k, v) x (dil + ring + sink rows)

    const uint8_t *src_k = static_cast<const uint8_t *>(p.k) + (size_t)bh * p.T * row_bytes;
    const uint8_t *src_v = static_cast<const uint8_t *>(p.v) + (size_t)bh * p.T * row_bytes;
    // job -> (source row, destination row) of this (b, h)
    auto locate = [&](long long job, const uint8_t *&src, uint8_t *&dst) {
        const bool is_v = job >= per;
        const long long r = is_v ? job - per : job;
        long long pos;
        if (r < n_dil) {
            const long long i = i_lo + r;
            pos = i * D + D - 1;
            uint8_t *base = static_cast<uint8_t *>(is_v ? p.vdil : p.kdil);
            if constexpr (PAGED) {
                const int32_t pg = p.page_table[(size_t)bhc * p.max_pages + (i >> p.page_shift)];
                if ((uint32_t)pg < (uint32_t)p.n_pages) {
                    dst = base + (((size_t)pg << p.page_shift) + (size_t)(i & ((1ll << p.page_shift) - 1))) * row_bytes;
                } else {
                    dst = nullptr;                      // no such page: skipped, error recorded
                    record_error(p.hdr, RAT_ERR_INVALID, 0x500u);
                }
            } else {
                dst = base + ((size_t)b * p.total_cap + p.off[h] + i) * row_bytes;
            }
        } else if (r < n_dil + n_ring) {
            pos = r_lo + (r - n_dil);
            uint8_t *base = static_cast<uint8_t *>(is_v ? p.vwin : p.kwin);
            dst = base + ((size_t)bhc * p.W + (size_t)(pos % p.W)) * row_bytes;
        } else {
            pos = p.pos0 + (r - n_dil - n_ring);
            uint8_t *base = static_cast<uint8_t *>(is_v ? p.vsink : p.ksink);
            dst = base + ((size_t)bhc * p.n_sink + (size_t)pos) * row_bytes;
        }
        src = (is_v ? src_v : src_k) + (size_t)(pos - p.pos0) * row_bytes;
    };
    // kU jobs per thread and trip, their loads issued together before the stores
    constexpr int kU = 4;
    const long long stride = (long long)nblk * rows_per_pass;
    for (long long base = (long long)blk * rows_per_pass + lane_r; base < njobs; base += kU * stride) {
        uint4 val[kU];
        uint8_t *dst[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const long long job = base + u * stride;
            dst[u] = nullptr;
            if (job < njobs) {
                const uint8_t *src;
                locate(job, src, dst[u]);
                if (!PAGED || dst[u]) val[u] = *reinterpret_cast<const uint4 *>(src + lane_c * 16);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u)
            if (dst[u]) *reinterpret_cast<uint4 *>(dst[u] + lane_c * 16) = val[u];
    }
    // recurrence state (float32), once per (b, h)
    if (blk == 0) {
        for (int c = threadIdx.x; c < p.d; c += blockDim.x) {
            if (p.hTk && p.hk != p.hTk) p.hk[(size_t)bhc * p.d + c] = p.hTk[(size_t)bh * p.d + c];
            if (p.hTv && p.hv != p.hTv) p.hv[(size_t)bhc * p.d + c] = p.hTv[(size_t)bh * p.d + c];
        }
        if (paged && p.seq_pos && h == 0 && threadIdx.x == 0) p.seq_pos[p.seq] = end;
    }
}

int launch_compress(const CompressParams &p_in, void *stream) {
    // CTAs per head: enough for about kU rows per thread, at least one (it copies the state)
    CompressParams p = p_in;
    const int rows_per_pass = 256 / (p.d * p.esize / 16);
    int acc = 0;
    for (int h = 0; h < p.H; ++h) {
        const long long D = p.Dh[h];
        const long long cap = p.page_table ? (long long)p.max_pages << p.page_shift : p.Tcap / D;
        const long long n_dil = std::max(0ll, std::min((p.pos0 + p.T) / D, cap) - p.pos0 / D);
        const long long n_ring = p.W > 0 ? std::min(p.W, p.T) : 0;     // the last min(W, T) positions
        const long long n_sk = std::max(0ll, std::min(p.pos0 + p.T, (long long)p.n_sink) - p.pos0);
        const long long jobs = 2 * (n_dil + n_ring + n_sk);
        long long n = (jobs + rows_per_pass * 4 - 1) / (rows_per_pass * 4);
        n = std::max(1ll, std::min(n, 4096ll));
        p.blk0[h] = acc;
        acc += (int)n;
    }
    p.blk0[p.H] = acc;
    const long long grid = (long long)acc * p.B;
    if (grid > 0x7fffffffll) return RAT_ERR_UNSUPPORTED;
    if (p.page_table) compress_kernel<true><<<(unsigned)grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    else compress_kernel<false><<<(unsigned)grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

}  // namespace rat
