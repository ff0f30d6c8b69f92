// rope_kernel.cuh -- the attention's prologue: split a packed QKV projection
// into q, k, v and apply the rotary embedding to q and k, in one pass.
//
// What it computes (inferencelayer "src/vision_gpu.rs", VIS_QKV_ROPE and its
// doc): the projection output is [T, 3*hid] per token (q | k | v, each H
// heads of D); the rope tables cos/sin are [T, D] f32, precomputed by the
// caller (a 2-D rope is a table built from the patch's row and column);
// per head
//     x'[d] = x[d] * cos[d] + rotate_half(x)[d] * sin[d],
//     rotate_half(x)[d] = -x[d + D/2] (d < D/2),  x[d - D/2] (d >= D/2),
// for q and k; v is copied.  Outputs are token-major [T, H, D], the layout
// the attention kernel reads.  With kCopyV = false v is neither read nor
// written: the attention then reads it straight out of the packed
// projection (token stride 3*H*D), and the prologue moves a third fewer bytes.
//
// The pass is pure HBM traffic (read 3*T*H*D elements and the tables, write
// 3*T*H*D elements), so the design is about coalescing.  A head's row takes
// `span` lanes (the power of two >= D/4), lane l of the span holding
// elements 4l..4l+3 (8-byte accesses, consecutive lanes consecutive
// addresses; lanes >= D/4 of the span idle): 32 lanes for D > 64, and for
// D <= 64 (kPair) 16, a warp then holding two consecutive heads of a token
// side by side, so that each load or store instruction moves 2*D*2
// contiguous bytes (256 at D = 64) instead of leaving half the warp idle.
// rotate_half's partner of element d is d +- D/2, which lives in lane
// l +- D/8 of the same span (D/2 is a multiple of 4): one warp shuffle.
// Arithmetic in f32 (one fma per element after the sin product), one
// rounding to the storage dtype.
#pragma once

#include <cstdint>

namespace vitattn {

constexpr int kRopeThreads = 256;

__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
    uint2 r;
    asm volatile("ld.global.nc.v2.b32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
__device__ __forceinline__ float4 ld_nc_f4(const void* p) {
    float4 r;
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ void st_v2(void* p, uint2 v) {
    asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// Two 16-bit values of a word, widened exactly to f32 (lo first).
template <bool kBF16>
__device__ __forceinline__ float2 unpack2(uint32_t u) {
    if (kBF16) return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    float2 r;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tcvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "r"(u));
    return r;
}
template <bool kBF16>
__device__ __forceinline__ uint32_t pack2rn(float lo, float hi) {
    uint32_t r;
    if (kBF16)
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    else
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// x*c + sign*p*s for four elements held as two 16-bit pairs.
template <bool kBF16>
__device__ __forceinline__ uint2 rotate4(uint2 x, uint2 p, float4 c, float4 s, float sign) {
    const float2 x0 = unpack2<kBF16>(x.x), x1 = unpack2<kBF16>(x.y);
    const float2 p0 = unpack2<kBF16>(p.x), p1 = unpack2<kBF16>(p.y);
    uint2 r;
    r.x = pack2rn<kBF16>(fmaf(x0.x, c.x, sign * p0.x * s.x), fmaf(x0.y, c.y, sign * p0.y * s.y));
    r.y = pack2rn<kBF16>(fmaf(x1.x, c.z, sign * p1.x * s.z), fmaf(x1.y, c.w, sign * p1.y * s.w));
    return r;
}

// Rows (heads) of one token a lane handles per loop trip: their loads are all
// issued before any is used (several rows in flight per warp), and the
// token's cos/sin row is loaded once for all of them.  Without the v copy a
// head holds two rows instead of three, so twice as many fit.
constexpr int kRopeHeadsPerWarp = 4;
__host__ __device__ constexpr int rope_heads_per_warp(bool copy_v) {
    return copy_v ? kRopeHeadsPerWarp : 2 * kRopeHeadsPerWarp;
}

// Heads a warp holds side by side: two (16 lanes each) when D <= 64.
__host__ __device__ constexpr bool rope_pair(int D) { return D <= 64; }
__host__ __device__ constexpr int rope_lane_groups(int D) { return rope_pair(D) ? 2 : 1; }

template <bool kBF16, bool kCopyV, bool kPair>
__global__ void __launch_bounds__(kRopeThreads, 4) qkv_rope_kernel(const uint8_t* __restrict__ qkv,
                                                                   const float* __restrict__ cs,
                                                                   const float* __restrict__ sn,
                                                                   uint8_t* __restrict__ q,
                                                                   uint8_t* __restrict__ k,
                                                                   uint8_t* __restrict__ v, long long T,
                                                                   int H, int D) {
    constexpr int R = rope_heads_per_warp(kCopyV);
    const int lane = threadIdx.x & 31;
    constexpr int span = kPair ? 16 : 32;  // lanes of one head's row
    constexpr int G = 32 / span;           // heads side by side in the warp
    const int grp = lane / span;           // this lane's head among them
    const int sl = lane % span;            // this lane's place in its head's row
    constexpr int per_trip = R * G;        // heads of a token per loop trip
    const int groups = (H + per_trip - 1) / per_trip;  // loop trips per token
    const long long items = T * (long long)groups;
    const long long stride = (long long)gridDim.x * (kRopeThreads / 32);
    const int active_lanes = D / 4;
    const int half_lanes = D / 8;
    const bool active = sl < active_lanes;
    const int partner = grp * span + (sl < half_lanes ? sl + half_lanes : sl - half_lanes);
    const float sign = sl < half_lanes ? -1.f : 1.f;
    const size_t hd2 = (size_t)H * (size_t)D * 2u;  // bytes of one token's q (or k, v) heads
    for (long long it = (long long)blockIdx.x * (kRopeThreads / 32) + (threadIdx.x >> 5); it < items;
         it += stride) {
        const long long t = it / groups;
        const int h0 = (int)(it - t * groups) * per_trip;
        const int nh = min(per_trip, H - h0);
        // row r of this lane is head h0 + r*G + grp; byte offsets of the lane's
        // 4 elements of row 0 in qkv and in the outputs
        const size_t in0 = (size_t)t * 3u * hd2 + ((size_t)(h0 + grp) * (size_t)D + 4u * (size_t)sl) * 2u;
        const size_t out0 = (size_t)t * hd2 + ((size_t)(h0 + grp) * (size_t)D + 4u * (size_t)sl) * 2u;
        const size_t head2 = (size_t)G * (size_t)D * 2u;  // from one row of the lane to the next
        float4 c = make_float4(0.f, 0.f, 0.f, 0.f), s = c;
        uint2 xq[R], xk[R], xv[R];
        if (active) {
            c = ld_nc_f4(cs + (size_t)t * (size_t)D + 4u * (size_t)sl);
            s = ld_nc_f4(sn + (size_t)t * (size_t)D + 4u * (size_t)sl);
        }
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
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const uint2 pq = make_uint2(__shfl_sync(0xffffffffu, xq[r].x, partner),
                                        __shfl_sync(0xffffffffu, xq[r].y, partner));
            const uint2 pk = make_uint2(__shfl_sync(0xffffffffu, xk[r].x, partner),
                                        __shfl_sync(0xffffffffu, xk[r].y, partner));
            if (active && r * G + grp < nh) {
                const size_t o = out0 + (size_t)r * head2;
                st_v2(q + o, rotate4<kBF16>(xq[r], pq, c, s, sign));
                st_v2(k + o, rotate4<kBF16>(xk[r], pk, c, s, sign));
                if (kCopyV) st_v2(v + o, xv[r]);
            }
        }
    }
}

}  // namespace vitattn
