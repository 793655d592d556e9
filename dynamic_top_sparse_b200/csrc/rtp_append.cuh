// Index keys of new tokens: kidx[b, g, pos_b + t] = W_k_idx[g] . k_pre[b, g, t]
// ("Full Attention Strikes Back", gist.science technical summary, Method
// section 2: the 16-dim projector acts on the key before RoPE).
#pragma once

#include "rtp_common.cuh"

namespace rtp {

// A CTA is 16 output dims x 16 chunks of 8 input dims: thread (j, c) holds
// W[g][j][8c .. 8c+7] in registers, reads the same 8 dims of each key (one
// 16- or 32-byte load, in flight together with its W load), and the 16
// chunks of an output dim are summed over 4 lane-xor steps.  A decode-time
// append (one token) is therefore one round trip to memory and a 4-step
// reduction; longer appends give each CTA a run of `tpc` tokens, loading
// APP_TOK of them at a time.
constexpr int APP_THREADS = R * (D / 8);   // 256
constexpr int APP_TOK = 8;

template <typename KT, typename IT>
__global__ void __launch_bounds__(APP_THREADS)
append_kernel(const KT *__restrict__ k_pre, const float *__restrict__ W,
              const int32_t *__restrict__ pos, IT *__restrict__ kidx, int H_kv, int T, int tpc,
              long long N_max, unsigned long long mask, uint32_t *status) {
    const int b = blockIdx.y / H_kv, g = blockIdx.y % H_kv;
    if (!((mask >> g) & 1ull)) return;
    // k_pre and pos may come from the previous kernel of the stream
    pdl_wait();
    pdl_trigger();
    const long long p0 = pos[b];
    if (p0 < 0 || p0 + T > N_max) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, RTP_ERR_DEVICE_ARG);
        return;
    }
    const int j = threadIdx.x >> 4, c = threadIdx.x & 15;
    float w[8];
    {
        const float4 *wp = reinterpret_cast<const float4 *>(W + ((size_t)g * R + j) * D + 8 * c);
        const float4 lo = __ldg(wp), hi = __ldg(wp + 1);
        w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
        w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
    }
    const size_t bg = (size_t)b * H_kv + g;
    const int t_lo = blockIdx.x * tpc, t_hi = min(T, t_lo + tpc);
    for (int t0 = t_lo; t0 < t_hi; t0 += APP_TOK) {
        float kx[APP_TOK][8];
#pragma unroll
        for (int i = 0; i < APP_TOK; ++i) {
            const int t = min(t0 + i, t_hi - 1);      // the tail re-reads its last token
            Row<KT>::load8(k_pre + (bg * T + t) * D + 8 * c, kx[i]);
        }
#pragma unroll
        for (int i = 0; i < APP_TOK; ++i) {
            float s = w[0] * kx[i][0];
#pragma unroll
            for (int e = 1; e < 8; ++e) s = fmaf(w[e], kx[i][e], s);
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (c == 0 && t0 + i < t_hi) kidx[(bg * N_max + p0 + t0 + i) * R + j] = Row<IT>::from_float(s);
        }
    }
}

}  // namespace rtp
