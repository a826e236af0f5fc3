// attn_sm100.cu -- bf16 dilated attention prefill (tensor-core path; under construction).
#include <cstring>

#include "common.cuh"

namespace rat {

int launch_attn_sm100(const AttnSm100Args &a, void *stream) {
    AttnSimtParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = a.q; p.k = a.k; p.v = a.v; p.o = a.o;
    p.B = a.B; p.H = a.H; p.T = a.T; p.d = a.d; p.W = a.W;
    p.pos0 = a.pos0; p.rope = a.rope; p.scale_log2 = a.scale_log2;
    for (int h = 0; h < a.H; ++h) p.Dh[h] = a.Dh[h];
    for (int c = 0; c < 64; ++c) p.theta[c] = a.theta[c];
    return launch_attn_simt(p, RAT_BF16, stream);
}

}  // namespace rat
