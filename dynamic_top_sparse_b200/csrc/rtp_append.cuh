// Index keys of new tokens: kidx[b, g, pos_b + t] = W_k_idx[g] . k_pre[b, g, t]
// ("Full Attention Strikes Back", gist.science technical summary, Method
// section 2: the 16-dim projector acts on the key before RoPE).
#pragma once

#include "rtp_common.cuh"

namespace rtp {

constexpr int APP_WARPS = 8;   // tokens per CTA

template <typename KT, typename IT>
__global__ void __launch_bounds__(APP_WARPS * 32)
append_kernel(const KT *__restrict__ k_pre, const float *__restrict__ W,
              const int32_t *__restrict__ pos, IT *__restrict__ kidx, int H_kv, int T,
              long long N_max, unsigned long long mask, uint32_t *status) {
    __shared__ __align__(16) float Ws[R][D];
    const int b = blockIdx.y / H_kv, g = blockIdx.y % H_kv;
    if (!((mask >> g) & 1ull)) return;
    const long long p0 = pos[b];
    if (p0 < 0 || p0 + T > N_max) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, RTP_ERR_DEVICE_ARG);
        return;
    }
    for (int i = threadIdx.x; i < R * D / 4; i += blockDim.x)
        reinterpret_cast<float4 *>(&Ws[0][0])[i] = __ldg(reinterpret_cast<const float4 *>(W + (size_t)g * R * D) + i);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * APP_WARPS + warp;
    if (t >= T) return;
    const size_t bg = (size_t)b * H_kv + g;
    float kx[4];
    Row<KT>::load4(k_pre + (bg * T + t) * D + lane * 4, kx);
    float mine = 0.0f;
#pragma unroll
    for (int j = 0; j < R; ++j) {
        const float4 w = *reinterpret_cast<const float4 *>(&Ws[j][lane * 4]);
        float s = w.x * kx[0];
        s = fmaf(w.y, kx[1], s);
        s = fmaf(w.z, kx[2], s);
        s = fmaf(w.w, kx[3], s);
        s = warp_sum(s);
        if (lane == j) mine = s;
    }
    if (lane < R) kidx[(bg * N_max + p0 + t) * R + lane] = Row<IT>::from_float(mine);
}

}  // namespace rtp
