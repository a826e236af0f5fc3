// attn_simt.cu -- causal dilated attention on CUDA cores (float32 path; any d in {64, 128}).
//
// RAT+ abstract and "RAT+ Deep Dive" sections 3.1 and 6: query t of head h attends to
//   S(t) = { t-We < j <= t }  U  { j <= t-We : j mod D_h = D_h - 1 },   We = max(W, 1),
// the local window (self included) and the chunk ends older than it; with n_sink > 0 also the
// first n_sink positions (StreamingLLM's attention sinks, section 6's layer-wise hybrid), each
// key once; with top_k > 0 also every position of the top_k chunks wholly older than the window,
// a chunk [cD, cD + D - 1] scored by its chunk-end key (section 4: dilation combined with top-k
// selection; ties go to the earlier chunk).  This kernel is also the path for every call with
// sinks or top-k.  One warp per query:
// each lane holds d/32 channels of the query and of the running output; for every key of
// S(t) the warp reduces the dot product with shuffles and applies an online softmax in
// float32 (exp2 with the scale folded in).  Keys are visited in groups of four so four row
// loads are in flight at once.  This is the float32 production path (a tensor-core bf16 or
// tf32 product would not meet float32 accuracy) and a readable GPU statement of the mask.
#include "common.cuh"

namespace rat {

constexpr int kMaxTopK = 16;

template <typename E, int DH>
__global__ void __launch_bounds__(256) attn_simt_kernel(const __grid_constant__ AttnSimtParams p) {
    __shared__ int s_sel[8][kMaxTopK];          // selected chunks of each warp's query
    constexpr int CPL = DH / 32;
    constexpr int EB = sizeof(E);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, h = bh % p.H;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= p.T) return;
    const int D = p.Dh[h];
    const int We = p.W > 1 ? p.W : 1;
    const uint8_t *kb = static_cast<const uint8_t *>(p.k) + (size_t)bh * p.T * DH * EB + lane * CPL * EB;
    const uint8_t *vb = static_cast<const uint8_t *>(p.v) + (size_t)bh * p.T * DH * EB + lane * CPL * EB;
    const size_t qoff = ((size_t)bh * p.T + t) * DH * EB + lane * CPL * EB;

    float q[CPL];
    RowIO<E, CPL>::load(static_cast<const uint8_t *>(p.q) + qoff, q);
    if (p.rope) {
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            const int c = lane * CPL + j;
            float cs, sn;
            rope_cs(p.pos0 + t, p.theta[c % (DH / 2)], cs, sn);
            const float partner = __shfl_xor_sync(0xffffffffu, q[j], 16);
            q[j] = c < DH / 2 ? q[j] * cs - partner * sn : q[j] * cs + partner * sn;
        }
    }
    float m = -INFINITY, l = 0.f, o[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) o[j] = 0.f;

    // the key list: window positions first, then the chunk ends older than the window, then
    // the sinks older than the window that are not chunk ends (sink s is position
    // s + s / (D-1): the D-1 non-chunk-ends of each chunk in turn)
    const int w_lo = max(0, t - We + 1);
    const int n_win = t - w_lo + 1;
    const int n_dil = t - We + 1 >= D ? (t - We + 1) / D : 0;   // j = D-1, .., n_dil*D - 1 <= t-We
    const int s_lim = min(p.n_sink, max(0, t - We + 1));
    const int n_snk = D > 1 ? s_lim - s_lim / D : 0;
    const int n_base = n_win + n_dil + n_snk;
    // top-k: score every candidate chunk by its chunk-end key; every lane keeps the same list of
    // the kMaxTopK best (score descending, then chunk ascending) by carrying each new candidate
    // down the list
    int n_sel = 0;
    if (p.top_k > 0 && n_dil > 0 && D > 1) {
        float bs[kMaxTopK];
        int bc[kMaxTopK];
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i) { bs[i] = -INFINITY; bc[i] = 0x7fffffff; }
        for (int c = 0; c < n_dil; ++c) {
            float kx[CPL];
            RowIO<E, CPL>::load(kb + (size_t)(c * D + D - 1) * DH * EB, kx);
            float dot = 0.f;
#pragma unroll
            for (int j = 0; j < CPL; ++j) dot = fmaf(q[j], kx[j], dot);
            float cs = warp_sum(dot);
            int cc = c;
#pragma unroll
            for (int i = 0; i < kMaxTopK; ++i) {
                if (cs > bs[i] || (cs == bs[i] && cc < bc[i])) {
                    const float ts = bs[i];
                    const int tc = bc[i];
                    bs[i] = cs;
                    bc[i] = cc;
                    cs = ts;
                    cc = tc;
                }
            }
        }
        n_sel = min(p.top_k, n_dil);
        if (lane == 0) {
#pragma unroll
            for (int i = 0; i < kMaxTopK; ++i) s_sel[warp][i] = bc[i];
        }
        __syncwarp();
    }
    const int n = n_base + n_sel * (D - 1);
    for (int base = 0; base < n; base += 4) {
        float kx[4][CPL], vx[4][CPL];
        bool ok[4];
        int cnt = min(4, n - base);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int idx = base + u;
            ok[u] = u < cnt;
            if (u < cnt) {
                int j;
                if (idx < n_win) j = w_lo + idx;
                else if (idx < n_win + n_dil) j = (idx - n_win) * D + D - 1;
                else if (idx < n_base) {
                    const int s = idx - n_win - n_dil;
                    j = s + s / (D - 1);
                } else {                               // a position of a selected chunk
                    const int e = idx - n_base;
                    j = s_sel[warp][e / (D - 1)] * D + e % (D - 1);
                    ok[u] = j >= p.n_sink;             // sinks are listed already
                }
                RowIO<E, CPL>::load(kb + (size_t)j * DH * EB, kx[u]);
                RowIO<E, CPL>::load(vb + (size_t)j * DH * EB, vx[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (ok[u]) {
                float dot = 0.f;
#pragma unroll
                for (int j = 0; j < CPL; ++j) dot = fmaf(q[j], kx[u][j], dot);
                const float s = warp_sum(dot) * p.scale_log2;
                const float mn = fmaxf(m, s);
                const float corr = exp2f(m - mn);
                const float pj = exp2f(s - mn);
                l = fmaf(l, corr, pj);
#pragma unroll
                for (int j = 0; j < CPL; ++j) o[j] = fmaf(o[j], corr, pj * vx[u][j]);
                m = mn;
            }
        }
    }
    const float inv = 1.0f / l;
#pragma unroll
    for (int j = 0; j < CPL; ++j) o[j] *= inv;
    RowIO<E, CPL>::store(static_cast<uint8_t *>(p.o) + qoff, o);
    if (p.lse && lane == 0) p.lse[(size_t)bh * p.T + t] = m + log2f(l);
}

int launch_attn_simt(const AttnSimtParams &p, int dtype, void *stream) {
    dim3 grid((unsigned)((p.T + 7) / 8), (unsigned)(p.B * p.H));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == RAT_F32) {
        if (p.d == 64) attn_simt_kernel<float, 64><<<grid, 256, 0, s>>>(p);
        else attn_simt_kernel<float, 128><<<grid, 256, 0, s>>>(p);
    } else {
        if (p.d == 64) attn_simt_kernel<__nv_bfloat16, 64><<<grid, 256, 0, s>>>(p);
        else attn_simt_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>(p);
    }
    return cudaGetLastError() == cudaSuccess ? RAT_OK : RAT_ERR_CUDA;
}

}  // namespace rat
