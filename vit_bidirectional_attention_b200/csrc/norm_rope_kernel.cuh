// norm_rope_kernel.cuh -- the attention's prologue with a per-head RMS norm
// of q and k ahead of the rotary embedding.
//
// What it computes (inferencelayer "src/vision_gpu.rs", GLM_QKV_QKNORM_ROPE
// and its doc, GLM-OCR vision tower): as qkv_rope_kernel, except that each
// head's q row x (and k row) is first normalised over its D elements,
//     y[d] = x[d] / sqrt(mean_e x[e]^2 + eps) * w[d],
// with one weight vector w[D] for q and another for k, shared by all heads;
// the rotation is then applied to y (norm first, rope second).  v is copied.
//
// Same thread layout as qkv_rope_kernel: one warp per (token, head), lane l
// holding elements 4l..4l+3.  The head's sum of squares is a butterfly over
// the warp (idle lanes hold zeros; a + b == b + a, so every lane ends with the
// same sum), the rotation partner d +- D/2 is one shuffle away as before, and
// both its weights and this lane's are loaded once per warp.  The norm costs
// two f32 roundings (IEEE sqrt and divide) per head row; the extra traffic is
// the two weight vectors, read once per warp from L1/L2.
#pragma once

#include "rope_kernel.cuh"

namespace vitattn {

// Sum of the squares of four 16-bit elements, in f32.
template <bool kBF16>
__device__ __forceinline__ float sumsq4(uint2 x) {
    const float2 a = unpack2<kBF16>(x.x), b = unpack2<kBF16>(x.y);
    return fmaf(b.y, b.y, fmaf(b.x, b.x, fmaf(a.y, a.y, a.x * a.x)));
}

// y*c + sign*yp*s with y = x*inv*w and yp = p*inv*wp, for four elements.
template <bool kBF16>
__device__ __forceinline__ uint2 norm_rotate4(uint2 x, uint2 p, float inv, float4 w, float4 wp, float4 c,
                                              float4 s, float sign) {
    const float2 x0 = unpack2<kBF16>(x.x), x1 = unpack2<kBF16>(x.y);
    const float2 p0 = unpack2<kBF16>(p.x), p1 = unpack2<kBF16>(p.y);
    const float y0 = x0.x * inv * w.x, y1 = x0.y * inv * w.y, y2 = x1.x * inv * w.z, y3 = x1.y * inv * w.w;
    const float q0 = p0.x * inv * wp.x, q1 = p0.y * inv * wp.y, q2 = p1.x * inv * wp.z, q3 = p1.y * inv * wp.w;
    uint2 r;
    r.x = pack2rn<kBF16>(fmaf(y0, c.x, sign * q0 * s.x), fmaf(y1, c.y, sign * q1 * s.y));
    r.y = pack2rn<kBF16>(fmaf(y2, c.z, sign * q2 * s.z), fmaf(y3, c.w, sign * q3 * s.w));
    return r;
}

// Resident blocks per SM: the four weight vectors held per lane (16
// registers) lift a thread to 80 registers, so three 256-thread blocks fit
// (four would cap it at 64 and spill).  The grid is this many per SM.
constexpr int kNormRopeBlocksPerSm = 3;

template <bool kBF16>
__global__ void __launch_bounds__(kRopeThreads, kNormRopeBlocksPerSm) qkv_norm_rope_kernel(
    const uint8_t* __restrict__ qkv, const float* __restrict__ cs, const float* __restrict__ sn,
    const float* __restrict__ qw, const float* __restrict__ kw, float eps, uint8_t* __restrict__ q,
    uint8_t* __restrict__ k, uint8_t* __restrict__ v, long long T, int H, int D) {
    constexpr int R = kRopeHeadsPerWarp;
    const int lane = threadIdx.x & 31;
    const int groups = (H + R - 1) / R;
    const long long items = T * (long long)groups;
    const long long stride = (long long)gridDim.x * (kRopeThreads / 32);
    const int active_lanes = D / 4;
    const int half_lanes = D / 8;
    const bool active = lane < active_lanes;
    const int partner = lane < half_lanes ? lane + half_lanes : lane - half_lanes;
    const float sign = lane < half_lanes ? -1.f : 1.f;
    const float fd = (float)D;
    const size_t hd2 = (size_t)H * (size_t)D * 2u;
    float4 wq = make_float4(0.f, 0.f, 0.f, 0.f), wqp = wq, wk = wq, wkp = wq;
    if (active) {  // partner < active_lanes whenever lane is active
        wq = ld_nc_f4(qw + 4 * lane);
        wqp = ld_nc_f4(qw + 4 * partner);
        wk = ld_nc_f4(kw + 4 * lane);
        wkp = ld_nc_f4(kw + 4 * partner);
    }
    for (long long it = (long long)blockIdx.x * (kRopeThreads / 32) + (threadIdx.x >> 5); it < items;
         it += stride) {
        const long long t = it / groups;
        const int h0 = (int)(it - t * groups) * R;
        const int nh = min(R, H - h0);
        const size_t in0 = (size_t)t * 3u * hd2 + ((size_t)h0 * (size_t)D + 4u * (size_t)lane) * 2u;
        const size_t out0 = (size_t)t * hd2 + ((size_t)h0 * (size_t)D + 4u * (size_t)lane) * 2u;
        const size_t head2 = (size_t)D * 2u;
        float4 c = make_float4(0.f, 0.f, 0.f, 0.f), s = c;
        uint2 xq[R], xk[R], xv[R];
        if (active) {
            c = ld_nc_f4(cs + (size_t)t * (size_t)D + 4u * (size_t)lane);
            s = ld_nc_f4(sn + (size_t)t * (size_t)D + 4u * (size_t)lane);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            xq[r] = xk[r] = xv[r] = make_uint2(0u, 0u);
            if (active && r < nh) {
                const uint8_t* src = qkv + in0 + (size_t)r * head2;
                xq[r] = ld_nc_v2(src);
                xk[r] = ld_nc_v2(src + hd2);
                xv[r] = ld_nc_v2(src + 2u * hd2);
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float sq = sumsq4<kBF16>(xq[r]), sk = sumsq4<kBF16>(xk[r]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
            }
            const float iq = 1.f / sqrtf(sq / fd + eps), ik = 1.f / sqrtf(sk / fd + eps);
            const uint2 pq = make_uint2(__shfl_sync(0xffffffffu, xq[r].x, partner),
                                        __shfl_sync(0xffffffffu, xq[r].y, partner));
            const uint2 pk = make_uint2(__shfl_sync(0xffffffffu, xk[r].x, partner),
                                        __shfl_sync(0xffffffffu, xk[r].y, partner));
            if (active && r < nh) {
                const size_t o = out0 + (size_t)r * head2;
                st_v2(q + o, norm_rotate4<kBF16>(xq[r], pq, iq, wq, wqp, c, s, sign));
                st_v2(k + o, norm_rotate4<kBF16>(xk[r], pk, ik, wk, wkp, c, s, sign));
                st_v2(v + o, xv[r]);
            }
        }
    }
}

}  // namespace vitattn
