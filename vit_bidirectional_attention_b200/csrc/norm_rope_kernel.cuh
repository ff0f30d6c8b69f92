// norm_rope_kernel.cuh -- the attention's prologue with a per-head RMS norm
// of q and k ahead of the rotary embedding.
//
// What it computes (inferencelayer "src/vision_gpu.rs", GLM_QKV_QKNORM_ROPE
// and its doc, GLM-OCR vision tower): as qkv_rope_kernel, except that each
// head's q row x (and k row) is first normalised over its D elements,
//     y[d] = x[d] / sqrt(mean_e x[e]^2 + eps) * w[d],
// with one weight vector w[D] for q and another for k, shared by all heads;
// the rotation is then applied to y (norm first, rope second).  v is copied
// (kCopyV), or left in the packed projection for the attention to read there.
//
// Same thread layout as qkv_rope_kernel: a head's row on `span` lanes, lane l
// of the span holding elements 4l..4l+3, 32 / span heads side by side.
// Since the norm is one factor per head row,
//     x'[d] = inv * (x[d] * A[d] + p[d] * B[d]),
//     A[d] = w[d] * cos[d],  B[d] = sign(d) * w[p(d)] * sin[d],
// with p the rotation partner d +- D/2 and inv = 1/sqrt(mean x^2 + eps): A
// and B are formed once per token (from the weights, re-read from L1, and
// the token's table row) and serve all its heads, leaving two multiplies
// and an fma per element.  The head's sum of squares is an xor butterfly
// over the lanes the head occupies (lanes past D/4 inside that power of two
// hold zeros, and the butterfly's offsets stay inside the span; a + b == b + a,
// so every lane of the head ends with the same sum); the
// inverse root is rsqrtf of one fma (mean plus eps).  The extra traffic is
// the two weight vectors, read per token from L1.
#pragma once

#include "rope_kernel.cuh"

namespace vitattn {

// Sum of the squares of four 16-bit elements, in f32.
template <bool kBF16>
__device__ __forceinline__ float sumsq4(uint2 x) {
    const float2 a = unpack2<kBF16>(x.x), b = unpack2<kBF16>(x.y);
    return fmaf(b.y, b.y, fmaf(b.x, b.x, fmaf(a.y, a.y, a.x * a.x)));
}

__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
    return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}

// inv * (x*A + p*B) for four elements.
template <bool kBF16>
__device__ __forceinline__ uint2 norm_rotate4(uint2 x, uint2 p, float inv, float4 A, float4 B) {
    const float2 x0 = unpack2<kBF16>(x.x), x1 = unpack2<kBF16>(x.y);
    const float2 p0 = unpack2<kBF16>(p.x), p1 = unpack2<kBF16>(p.y);
    uint2 r;
    r.x = pack2rn<kBF16>(inv * fmaf(x0.x, A.x, p0.x * B.x), inv * fmaf(x0.y, A.y, p0.y * B.y));
    r.y = pack2rn<kBF16>(inv * fmaf(x1.x, A.z, p1.x * B.z), inv * fmaf(x1.y, A.w, p1.y * B.w));
    return r;
}

// Resident blocks per SM (the grid is this many per SM).
constexpr int kNormRopeBlocksPerSm = 3;

template <bool kBF16, bool kCopyV, bool kPair>
__global__ void __launch_bounds__(kRopeThreads, kNormRopeBlocksPerSm) qkv_norm_rope_kernel(
    const uint8_t* __restrict__ qkv, const float* __restrict__ cs, const float* __restrict__ sn,
    const float* __restrict__ qw, const float* __restrict__ kw, float eps, uint8_t* __restrict__ q,
    uint8_t* __restrict__ k, uint8_t* __restrict__ v, long long T, int H, int D) {
    constexpr int R = kRopeHeadsPerWarp;
    const int lane = threadIdx.x & 31;
    constexpr int span = kPair ? 16 : 32;  // lanes of a head's row (and of its butterfly)
    constexpr int G = 32 / span;           // heads side by side in the warp
    const int grp = lane / span;
    const int sl = lane % span;
    constexpr int per_trip = R * G;
    const int groups = (H + per_trip - 1) / per_trip;
    const long long items = T * (long long)groups;
    const long long stride = (long long)gridDim.x * (kRopeThreads / 32);
    const int active_lanes = D / 4;
    const int half_lanes = D / 8;
    const bool active = sl < active_lanes;
    const int psl = sl < half_lanes ? sl + half_lanes : sl - half_lanes;  // the partner's place in the row
    const int partner = grp * span + psl;
    const float sign = sl < half_lanes ? -1.f : 1.f;
    const float inv_d = 1.f / (float)D;
    const size_t hd2 = (size_t)H * (size_t)D * 2u;
    for (long long it = (long long)blockIdx.x * (kRopeThreads / 32) + (threadIdx.x >> 5); it < items;
         it += stride) {
        const long long t = it / groups;
        const int h0 = (int)(it - t * groups) * per_trip;
        const int nh = min(per_trip, H - h0);
        // row r of this lane is head h0 + r*G + grp
        const size_t in0 = (size_t)t * 3u * hd2 + ((size_t)(h0 + grp) * (size_t)D + 4u * (size_t)sl) * 2u;
        const size_t out0 = (size_t)t * hd2 + ((size_t)(h0 + grp) * (size_t)D + 4u * (size_t)sl) * 2u;
        const size_t head2 = (size_t)G * (size_t)D * 2u;
        uint2 xq[R], xk[R], xv[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            xq[r] = xk[r] = xv[r] = make_uint2(0u, 0u);
            if (active && r * G + grp < nh) {
                const uint8_t* src = qkv + in0 + (size_t)r * head2;
                xq[r] = ld_nc_v2(src);
                xk[r] = ld_nc_v2(src + hd2);
                if (kCopyV) xv[r] = ld_nc_v2(src + 2u * hd2);
            }
        }
        float4 Aq = make_float4(0.f, 0.f, 0.f, 0.f), Bq = Aq, Ak = Aq, Bk = Aq;
        if (active) {  // psl < D/4 whenever this lane is active
            const float4 c = ld_nc_f4(cs + (size_t)t * (size_t)D + 4u * (size_t)sl);
            const float4 s = ld_nc_f4(sn + (size_t)t * (size_t)D + 4u * (size_t)sl);
            const float4 ss = make_float4(sign * s.x, sign * s.y, sign * s.z, sign * s.w);
            Aq = mul4(ld_nc_f4(qw + 4 * sl), c);
            Bq = mul4(ld_nc_f4(qw + 4 * psl), ss);
            Ak = mul4(ld_nc_f4(kw + 4 * sl), c);
            Bk = mul4(ld_nc_f4(kw + 4 * psl), ss);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float sq = sumsq4<kBF16>(xq[r]), sk = sumsq4<kBF16>(xk[r]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                if (o < span) {  // warp-uniform
                    sq += __shfl_xor_sync(0xffffffffu, sq, o);
                    sk += __shfl_xor_sync(0xffffffffu, sk, o);
                }
            }
            const float iq = rsqrtf(fmaf(sq, inv_d, eps)), ik = rsqrtf(fmaf(sk, inv_d, eps));
            const uint2 pq = make_uint2(__shfl_sync(0xffffffffu, xq[r].x, partner),
                                        __shfl_sync(0xffffffffu, xq[r].y, partner));
            const uint2 pk = make_uint2(__shfl_sync(0xffffffffu, xk[r].x, partner),
                                        __shfl_sync(0xffffffffu, xk[r].y, partner));
            if (active && r * G + grp < nh) {
                const size_t o = out0 + (size_t)r * head2;
                st_v2(q + o, norm_rotate4<kBF16>(xq[r], pq, iq, Aq, Bq));
                st_v2(k + o, norm_rotate4<kBF16>(xk[r], pk, ik, Ak, Bk));
                if (kCopyV) st_v2(v + o, xv[r]);
            }
        }
    }
}

}  // namespace vitattn
