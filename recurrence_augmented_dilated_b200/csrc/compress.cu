// compress.cu -- build / extend the D-fold compressed KV cache from recurrence outputs.
//
// RAT+ abstract: dilation keeps every D-th key, which cuts the KV cache D-fold; the local
// window keeps the W most recent positions.  For the T new positions pos0 .. pos0+T-1 of every
// (b, h) this kernel copies
//   - each chunk end p = i*D_h + D_h - 1 (i < cap_h) to dil entry i of head h, and
//   - each of the last min(W, T) positions p to ring slot p mod W,
// for k~ and v~, bit for bit; and copies the final recurrence state into the cache.
// One CTA per (row block, b*h); 16-byte vector copies, one row per LPR lanes.
#include "common.cuh"

namespace rat {

__global__ void __launch_bounds__(256) compress_kernel(const __grid_constant__ CompressParams p) {
    const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
    const long long D = p.Dh[h];
    const long long cap = p.Tcap / D;
    const long long end = p.pos0 + p.T;
    const long long i_lo = p.pos0 / D;                       // first chunk end >= pos0
    const long long i_hi = min(end / D, cap);                // chunk ends < end, within capacity
    const long long n_dil = max(0ll, i_hi - i_lo);
    const long long r_lo = max(p.pos0, end - (long long)p.W);  // ring positions [r_lo, end)
    const long long n_ring = p.W > 0 ? end - r_lo : 0;
    const int row_bytes = p.d * p.esize;
    const int lpr = row_bytes / 16;                          // lanes per row
    const int rows_per_pass = blockDim.x / lpr;
    const int lane_r = threadIdx.x / lpr, lane_c = threadIdx.x % lpr;
    const long long njobs = 2 * (n_dil + n_ring);            // (k, v) x (dil rows + ring rows)

    const uint8_t *src_k = static_cast<const uint8_t *>(p.k) + (size_t)bh * p.T * row_bytes;
    const uint8_t *src_v = static_cast<const uint8_t *>(p.v) + (size_t)bh * p.T * row_bytes;
    for (long long job = (long long)blockIdx.x * rows_per_pass + lane_r; job < njobs;
         job += (long long)gridDim.x * rows_per_pass) {
        const bool is_v = job >= n_dil + n_ring;
        const long long r = is_v ? job - (n_dil + n_ring) : job;
        long long pos;
        uint8_t *dst;
        if (r < n_dil) {
            const long long i = i_lo + r;
            pos = i * D + D - 1;
            uint8_t *base = static_cast<uint8_t *>(is_v ? p.vdil : p.kdil);
            dst = base + ((size_t)b * p.total_cap + p.off[h] + i) * row_bytes;
        } else {
            pos = r_lo + (r - n_dil);
            uint8_t *base = static_cast<uint8_t *>(is_v ? p.vwin : p.kwin);
            dst = base + (((size_t)b * p.H + h) * p.W + (size_t)(pos % p.W)) * row_bytes;
        }
        const uint8_t *src = (is_v ? src_v : src_k) + (size_t)(pos - p.pos0) * row_bytes;
        const uint4 val = *reinterpret_cast<const uint4 *>(src + lane_c * 16);
        *reinterpret_cast<uint4 *>(dst + lane_c * 16) = val;
    }
    // recurrence state (float32), once per (b, h)
    if (blockIdx.x == 0) {
        for (int c = threadIdx.x; c < p.d; c += blockDim.x) {
            if (p.hTk && p.hk != p.hTk) p.hk[(size_t)bh * p.d + c] = p.hTk[(size_t)bh * p.d + c];
            if (p.hTv && p.hv != p.hTv) p.hv[(size_t)bh * p.d + c] = p.hTv[(size_t)bh * p.d + c];
        }
    }
}

int launch_compress(const CompressParams &p, void *stream) {
    // enough CTAs per (b, h) to cover its dil rows in a few passes
    long long max_rows = 0;
    for (int h = 0; h < p.H; ++h) {
        const long long D = p.Dh[h];
        const long long n = min((p.pos0 + p.T) / D, p.Tcap / D) - p.pos0 / D;
        max_rows = n > max_rows ? n : max_rows;
    }
    max_rows = 2 * (max_rows + p.W);
    const int rows_per_pass = 256 / (p.d * p.esize / 16);
    long long gx = (max_rows + rows_per_pass * 4 - 1) / (rows_per_pass * 4);
    if (gx < 1) gx = 1;
    if (gx > 1024) gx = 1024;
    dim3 grid((unsigned)gx, (unsigned)(p.B * p.H));
    compress_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

}  // namespace rat
