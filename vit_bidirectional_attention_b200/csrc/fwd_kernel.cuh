// fwd_kernel.cuh -- sm_100a forward kernel of multi-head attention (no mask
// by default; cross lengths, the aligned causal mask, grouped-query heads,
// ragged batches and token-strided inputs are variants of the same body).
//
// A work item is one (batch b, head h) pair and up to two 128-row query tiles
// of it (256 query rows); a CTA runs one item, or loops over items.  K and V
// stream through a shared-memory ring in blocks of 128 keys.  Per key block j
// and query tile t:
//
//   S_t   = Q_t K_j^T                    tcgen05.mma, A = Q (smem), B = K (smem), f32 in TMEM
//   P_t   = exp2(S_t * c - m_t)          softmax warpgroup t, one thread per query row,
//                                        c = scale*log2(e); P rounded to f16 and written
//                                        back into TMEM over S_t
//   O_t  += P_t V_j                      tcgen05.mma, A = P (TMEM), B = V (smem), both f16,
//                                        f32 in TMEM
//
// with the running row maximum m_t, the row sum l_t and the rescaling of O_t
// kept exact in the online-softmax sense: O and l are always relative to the
// same (possibly stale) maximum, so the result is O/l at the end.  l_t sums the
// f32 probabilities before their rounding to f16 (within 2^-12 relative of
// the weights the P.V product uses).  A split item (a grid too small for two
// tiles per CTA) gives the two softmax warpgroups the two halves of ONE query
// tile's key blocks and merges their (m, l, O) at the end.
// The P.V product runs in f16 for both input dtypes: f16 has three more
// mantissa bits than bf16 for P.  For bf16 inputs V is converted to f16 in shared memory
// after it lands (exact for |v| < 2^16 apart from f16's subnormal range,
// below 2^-14, where the absolute error stays under 2^-25; larger |v| becomes
// inf and is reported by the checked entry point).  This is the
// online-softmax GEMM pair of inferencelayer "src/vision_gpu.rs" (doc of
// `vis_attn_coop_src`: "The obstacle, and the way round it"), except that the
// running output lives in tensor memory instead of being spilled to shared
// memory, and that it is only rescaled when a row maximum grows by more than
// 2^8 (the result is unchanged; probabilities stay <= 256, which bf16 and f16
// hold).  Keys past N are masked to probability 0 (same page, "Keys past the
// span ... are masked to zero probability").
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3    softmax for query tile 0 (TMEM lanes 0..127 through warp%4)
//   warps 4-7    softmax for query tile 1
//   warp  8      TMA producer (one lane) and TMEM allocator (whole warp)
//   warp  9      MMA issuer (one lane)
//   warps 10-11  bf16 inputs: convert each V block to f16 in shared memory
//                (f16 inputs: idle; they complete the third warpgroup)
// Registers: the launch gives every thread kLaunchRegs; the third warpgroup
// then gives most of its share back (setmaxnreg.dec to kSideRegs) and the two
// softmax warpgroups take it (setmaxnreg.inc to kSoftmaxRegs), so a softmax
// thread can hold its 128 scores and still keep many exponentials in flight.
//
// Work order.  The (tile, key block) units are numbered s = ntiles*j + t.
// Unit s gets S buffer s % NS, where NS = 3 S buffers fit in TMEM when
// DP <= 64 and 2 otherwise.  The MMA warp issues S for the first NS units,
// then for every unit s: O_t += P_s V_j, followed by S for unit s + NS in the
// buffer P_s has just been read from.  With NS = 3 a tile's next S is
// computed while its softmax still works on the current block; with NS = 2
// this is the classic two-tile ping-pong.  A looping CTA runs an item's
// epilogue after handing over the next item's first block.
//
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [128*b, 128*b+128)  S buffer b < NS, later P (16-bit pairs in its first 64 columns)
//   [128*NS + oc*t, ...)  O_t, DP of its oc = 64 (DP <= 64) or 128 columns used
//
// Shared memory: Q_0, Q_1 and a ring of kStages K/V slots, each a 128 x DP
// tile stored as column chunks of 64 / 32 / 16 elements (SW128 / SW64 / SW32
// swizzle, exactly as TMA writes them and as the MMA descriptors read them).
// DP is D rounded up to a multiple of 16; TMA zero-fills columns D..DP-1.
//
// Every wait is bounded by a time limit.  On expiry the kernel records a
// status code in g_vitattn_status, raises a CTA-wide abort flag that every
// other waiter polls, drains its own in-flight TMA copies and MMAs, frees its
// tensor memory and exits.
#pragma once

#include <cuda.h>

#include <cmath>
#include <cstdint>

#include "ptx.cuh"

// Kernel status words (this header is compiled into exactly one translation
// unit).  g_vitattn_status: 0, or a timeout code from a bounded in-kernel
// wait.  g_vitattn_range: nonzero once a bf16 V value of magnitude >= 2^16
// (outside f16's range) has been converted for the f16 P.V product.
__device__ unsigned int g_vitattn_status = 0;
__device__ unsigned int g_vitattn_range = 0;

namespace vitattn {

constexpr int kTileRows = 128;    // query rows per tile = TMEM lanes
constexpr int kBlockKeys = 128;   // keys per K/V block
constexpr int kTilesPerCta = 2;
constexpr int kMaxStages = 8;     // K/V ring slots at most (K in even slots, V in odd ones)
constexpr int kThreads = 384;
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kConvWarp = 10;  // first of the two V-converter warps
// Register split: 3 warps share each SMSP register file (16384 x 32-bit), so a
// 384-thread block launches at 168 per thread; 2*224 + 56 = 3*168 per SMSP and
// 256*224 + 128*56 = 384*168 per block: the reallocation never waits forever.
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 224;
constexpr uint32_t kSideRegs = 56;
static_assert(2 * kSoftmaxRegs + kSideRegs == 3 * kLaunchRegs, "register split per SMSP");
static_assert(256 * kSoftmaxRegs + 128 * kSideRegs == kThreads * kLaunchRegs, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when the max grows > 2^8

// Barrier indices inside the barrier array.
constexpr int kMaxQBufs = 2;
constexpr int kBarQFull = 0;                         // [kMaxQBufs][2 tiles] Q loaded
constexpr int kBarQEmpty = kBarQFull + 2 * kMaxQBufs; // [kMaxQBufs][2 tiles] last S read it
constexpr int kBarKvFull = kBarQEmpty + 2 * kMaxQBufs;  // [kMaxStages]
constexpr int kBarKvEmpty = kBarKvFull + kMaxStages; // [kMaxStages]
constexpr int kMaxSBufs = 3;
constexpr int kBarSFull = kBarKvEmpty + kMaxStages;  // [kMaxSBufs] one per S buffer
// [2 tiles][2] P written (and O rescaled) for blocks of even / odd index: with
// the S look-ahead a tile's softmax can finish block j+1 before the MMA warp
// has consumed block j, and one barrier per tile could then run two phases
// ahead of its waiter; block j+2 needs P.V of block j first, so two cannot.
constexpr int kBarPFull = kBarSFull + kMaxSBufs;
constexpr int kBarOReady = kBarPFull + 4;            // [2] per tile: a P.V product finished
constexpr int kBarOFull = kBarOReady + 2;            // [2] per tile: the item's last P.V finished
constexpr int kBarOEmpty = kBarOFull + 2;            // [2] per tile: the epilogue has read O
constexpr int kBarVReady = kBarOEmpty + 2;           // [kMaxStages / 2] bf16: the V slot's block is f16
constexpr int kBarDrain = kBarVReady + kMaxStages / 2;  // [1]
constexpr int kBarMerge = kBarDrain + 1;             // [1] split items: the upper key half's (m, l) are written
constexpr int kNumBars = kBarMerge + 1;

// Status codes written to g_vitattn_status (0 = fine).
constexpr unsigned kStatusTimeoutBase = 0x100;  // + site id

// Test-only flag: the producer skips its first V load so that the consumer's
// bounded wait runs out (exercises the timeout path without a fault).
constexpr int kFlagSkipFirstVLoad = 1;
// Test-only host flags: force two (or one) query tiles per CTA whatever the grid
// size; run the whole problem on at most three CTAs (many work items each).
constexpr int kFlagForceTwoTiles = 2;
constexpr int kFlagForceOneTile = 4;
constexpr int kFlagTinyGrid = 8;
// Test-only host flags: never split a query tile's key blocks over the two
// softmax warpgroups (see FwdParams::split), or split them from two key
// blocks on (by default from four: with fewer the merge costs what the
// shorter chain saves, measured on the 196-token block).
constexpr int kFlagNoSplit = 16;
constexpr int kFlagSplitFromTwo = 32;

// ---------------------------------------------------------------- column chunks

__host__ __device__ constexpr int chunk_count(int dp) {
    return dp / 64 + ((dp % 64) >= 32 ? 1 : 0) + ((dp % 32) != 0 ? 1 : 0);
}
__host__ __device__ constexpr int chunk_width(int dp, int c) {
    return c < dp / 64 ? 64 : ((c == dp / 64 && (dp % 64) >= 32) ? 32 : 16);
}
__host__ __device__ constexpr int chunk_col(int dp, int c) {
    int col = 0;
    for (int i = 0; i < c; ++i) col += chunk_width(dp, i);
    return col;
}
__host__ __device__ constexpr int width_class(int w) { return w == 64 ? 0 : (w == 32 ? 1 : 2); }
// tcgen05 shared-memory descriptor layout codes: SW128 = 2, SW64 = 4, SW32 = 6.
__host__ __device__ constexpr uint32_t swizzle_code(int w) { return w == 64 ? 2u : (w == 32 ? 4u : 6u); }

__host__ __device__ constexpr int tile_bytes(int dp) { return kTileRows * dp * 2; }
// TMEM: kTilesPerCta O accumulators of o_cols(dp) columns at the top, and as
// many 128-column S/P buffers below them as fit (3 when dp <= 64, else 2).
__host__ __device__ constexpr int o_cols(int dp) { return dp <= 64 ? 64 : 128; }
__host__ __device__ constexpr int s_buffers(int dp) {
    return (512 - kTilesPerCta * o_cols(dp)) / kBlockKeys;
}
// S buffers in use.  A third buffer is only used with two query tiles: then
// S for unit s is issued after P.V of unit s-3, so when tile t's softmax sees
// S(t, j) the product P.V(t, j-2) has finished, which is what makes the
// parity wait for P.V(t, j-1) in the O rescale unambiguous.  With one tile and
// three buffers only P.V(j-3) would be known complete.
__host__ __device__ constexpr int active_s_buffers(int ns, int ntiles) {
    return ntiles == 2 ? ns : (ns < 2 ? ns : 2);
}
// With ns buffers and ntiles tiles, S(t, j) is issued after P.V of unit
// ntiles*j + t - ns.  When that is P.V(t, j-1) itself (ns == ntiles), seeing
// S(t, j) already proves P.V(t, j-1) done and the separate "P.V done"
// barrier (one extra tcgen05.commit per product) is not needed.
__host__ __device__ constexpr bool pv_done_needed(int ns, int ntiles) { return ns != ntiles; }
// Q tiles are double-buffered (the next work item's Q loads while the current
// one runs) when a CTA loops over items and that fits in shared memory, i.e.
// up to DP = 112.
__host__ __device__ constexpr int q_buffers(int dp, bool loop) { return (loop && dp <= 112) ? 2 : 1; }
// K/V ring slots (even: K in even slots, V in odd ones).  Four hold two key
// blocks, each shared by the item's two tiles.  A split item's tiles read
// different blocks, so a step of both tiles fills four slots by itself: its
// ring is as deep as shared memory allows (eight slots up to DP = 80, six up
// to 112), so that the next step's blocks load during this one.
__host__ __device__ constexpr int kv_stages(int dp, bool split = false) {
    return split ? (dp <= 80 ? 8 : dp <= 112 ? 6 : 4) : 4;
}
static_assert(kMaxStages % 2 == 0, "K and V alternate in the ring");
static_assert(kv_stages(16, true) <= kMaxStages && kv_stages(128) <= kMaxStages, "ring barriers");
// Split items exchange one (m, l) pair per query row through shared memory.
constexpr int kMergeBytes = kTileRows * 2 * 4;
__host__ __device__ constexpr int smem_bytes(int dp, bool loop, bool split = false) {
    return (q_buffers(dp, loop) * kTilesPerCta + kv_stages(dp, split)) * tile_bytes(dp) + kNumBars * 8 + 16 +
           (split ? kMergeBytes : 0) + 1024;
}
// Every launchable configuration fits the 227 KB of dynamic shared memory a
// block may opt into.
__host__ __device__ constexpr bool smem_fits() {
    for (int dp = 16; dp <= 128; dp += 16)
        if (smem_bytes(dp, false) > 227 * 1024 || smem_bytes(dp, true) > 227 * 1024 ||
            smem_bytes(dp, false, true) > 227 * 1024)
            return false;
    return true;
}
static_assert(smem_fits(), "shared memory of every configuration");

// Ragged batches (several images' tokens packed along one axis, start
// offsets cu_seqlens): segment s is tokens start[s] .. start[s] + len[s] - 1,
// and its work items (head, group of query tiles) are item0[s] ..
// item0[s+1] - 1, qgroups[s] query groups per head.  The dense layout needs
// none of it (an empty table).
constexpr int kMaxSegs = 256;
template <bool kVarlen>
struct SegTable {
    int n;
};
template <>
struct SegTable<true> {
    int n;                    // segments
    int start[kMaxSegs];      // first token of segment s
    int len[kMaxSegs];        // its token count
    int qgroups[kMaxSegs];    // ceil(len / (128 * tiles_per_cta))
    int item0[kMaxSegs + 1];  // first work item of segment s; item0[n] = all items
};

struct alignas(64) FwdParams {
    CUtensorMap maps[3][3];  // [q, k, v][width class 64 / 32 / 16]
    void* out;
    long long out_ts;   // elements between consecutive tokens of out (H * D when dense)
    int B, N, H, D;
    int tiles_per_cta;  // query tiles a work item owns: 2, or 1 when 2 would leave SMs idle
    int n_qgroups;      // ceil(N / (128 * tiles_per_cta)): work items per (b, h) (dense layout)
    int n_items;        // all work items; a CTA takes items blockIdx.x + k * gridDim.x
    int n_kblocks;      // ceil(N / 128) (dense layout; a ragged batch takes it per segment)
    int kv_group;       // query heads per key/value head (1: multi-head; H / Hkv: grouped-query)
    int Nk;             // keys per (b, h), dense layout (N unless query and key lengths differ)
    int causal;         // nonzero: query i sees keys j <= i + causal_off only (aligned causal mask)
    int causal_off;     // Nk - N
    float* lse;         // optional [B, H, N] f32: log sum_j exp(scale * q_i . k_j); nullptr: not written
    int split;          // nonzero: a work item is ONE query tile whose key blocks are split in two halves,
                        // one per softmax warpgroup, merged at the end (grids too small to fill the SMs)
    float scale_log2;
    int flags;
    unsigned long long timeout_ns;
};

// ---------------------------------------------------------------- descriptors

// Shared-memory matrix descriptor (tcgen05): start address, leading and
// stride byte offsets (16-byte units), fixed version 1 at bit 46, layout code
// at bits 61..63.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                          uint32_t layout) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

// Instruction descriptor, kind::f16: f32 accumulator, A and B both bf16 (1) or
// both f16 (0), A K-major, B K-major (0) or MN-major (1), N >> 3, M >> 4.
__host__ __device__ constexpr uint32_t idesc_f16(bool bf16, int n, bool b_mn_major) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
           ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kTileRows >> 4) << 24);
}

// ---------------------------------------------------------------- bounded waits

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, unsigned site) {
    *abort_flag = 1;
    atomicCAS(&g_vitattn_status, 0u, kStatusTimeoutBase + site);
}

// Slow path of wait_one: spin with a time limit.
__device__ __forceinline__ bool wait_one_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           uint64_t timeout_ns, unsigned site) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > timeout_ns) {
            raise_abort(abort_flag, site);
            return false;
        }
    }
}

// One thread waits for the phase of `parity`; false on abort or timeout.
__device__ __forceinline__ bool wait_one(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t timeout_ns, unsigned site) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    return wait_one_slow(bar, parity, abort_flag, timeout_ns, site);
}

// Wait that ignores the abort flag, for draining in-flight work before exit.
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer_ns() - t0 > timeout_ns) return false;
    }
    return true;
}

// Slow path of wait_warp (whole warp, uniform outcome).
__device__ __forceinline__ bool wait_warp_slow(uint32_t bar, uint32_t parity, bool done,
                                            volatile int* abort_flag, uint64_t timeout_ns,
                                            unsigned site) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
        if (!done) done = ptx::mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, done)) return true;
        int give_up = 0;
        if ((threadIdx.x & 31) == 0) {
            if (*abort_flag) {
                give_up = 1;
            } else if (ptx::globaltimer_ns() - t0 > timeout_ns) {
                raise_abort(abort_flag, site);
                give_up = 1;
            }
        }
        if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
    }
}

// A whole warp waits; the outcome is uniform across the warp.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t timeout_ns, unsigned site) {
    const bool done = ptx::mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    return wait_warp_slow(bar, parity, done, abort_flag, timeout_ns, site);
}

// ---------------------------------------------------------------- softmax pieces

// Extreme of N values with 3-input min/max in a tree (compile-time shape, so
// every index is a constant and nothing leaves registers).
template <int N, bool kNeg>
__device__ __forceinline__ float tree3(const float* v) {
    if constexpr (N == 1) {
        return v[0];
    } else if constexpr (N == 2) {
        return kNeg ? fminf(v[0], v[1]) : fmaxf(v[0], v[1]);
    } else {
        constexpr int M = (N + 2) / 3;
        float t[M];
#pragma unroll
        for (int i = 0; i < M; ++i) {
            const float a = v[3 * i];
            const float b = 3 * i + 1 < N ? v[3 * i + 1] : a;
            const float c = 3 * i + 2 < N ? v[3 * i + 2] : a;
            t[i] = kNeg ? ptx::fmin3(a, b, c) : ptx::fmax3(a, b, c);
        }
        return tree3<M, kNeg>(t);
    }
}

// Row extreme of the raw scores in the direction that maximises c * s:
// max for c >= 0, min for c < 0.  Masked columns (>= valid) are skipped.
// Reduced 32 columns at a time so that few temporaries are live at once.
template <bool kPartial, bool kNeg>
__device__ __forceinline__ float row_extreme(const float (&s)[kBlockKeys], int valid) {
    const float fill = kNeg ? INFINITY : -INFINITY;
    float part[kBlockKeys / 32];
#pragma unroll
    for (int q = 0; q < kBlockKeys / 32; ++q) {
        float t[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) t[i] = (!kPartial || 32 * q + i < valid) ? s[32 * q + i] : fill;
        part[q] = tree3<32, kNeg>(t);
    }
    return tree3<kBlockKeys / 32, kNeg>(part);
}

// Pairs of exponentials (out of every 16 pairs) computed by the polynomial on
// the FMA/ALU pipes instead of ex2.approx on the MUFU pipe, which runs at 16
// results per clock per SM (f32 and f16 pairs alike, measured in the softmax
// loop) and is otherwise the softmax's bottleneck.
constexpr int kPolyPairs = 0;
__host__ __device__ constexpr bool poly_pair(int i) { return (i * kPolyPairs) % 16 < kPolyPairs; }

// 2^x for a pair, on the FMA and ALU pipes.  Cody-Waite style split
// x = j + f with j = round(x) (adding 1.5 * 2^23 leaves j in the low mantissa
// bits of t) and f in [-1/2, 1/2]; 2^f from a degree-3 minimax polynomial
// (Remez exchange on the relative error: max 7.5e-5, about a sixth of an f16
// ulp); j is then added to the exponent field.  x is clamped below at -125 so
// the exponent stays normal (such p round to 0 in f16 anyway).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    const float2 magic = make_float2(12582912.f, 12582912.f);
    const float2 t = ptx::fadd2(x, magic);
    const float2 f = ptx::fsub2(x, ptx::fsub2(t, magic));
    float2 p = ptx::ffma2(f, make_float2(0.0551716685f, 0.0551716685f),
                          make_float2(0.2426111251f, 0.2426111251f));
    p = ptx::ffma2(p, f, make_float2(0.6932609677f, 0.6932609677f));
    p = ptx::ffma2(p, f, make_float2(0.9999280572f, 0.9999280572f));
    return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// p = 2^(c*s - m) for one block, in f32 (ex2.approx, or the polynomial for
// some pairs), rounded to f16 and written to TMEM as f16 pairs at tP (64
// columns), 32 scores at a time.  x <= 8 here (the lazy rescale bound), so
// p <= 256; f16 keeps p down to 2^-24 (subnormals are kept).  Returns the sum
// of the f32 p (before rounding), kept in four f32 partial sums added two at
// a time (add.f32x2): the rounded weights the tensor core uses differ from
// these by at most 2^-12 relative each, so O / l is within 2^-12 relative of
// the weighted average of V rows with the rounded weights.  Summing the
// rounded halves instead (exact weights, one mixed-precision add each) costs
// 12-37% of the exponential throughput, measured.  Columns at or past `valid`
// get p = 0.
template <bool kPartial>
__device__ __forceinline__ float exp_pack_store(const float (&s)[kBlockKeys], int valid, float c2,
                                                float neg_m, uint32_t tP) {
    float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
#pragma unroll
    for (int q = 0; q < kBlockKeys / 32; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int c = 32 * q + 2 * i;
            const float2 x = ptx::ffma2(make_float2(s[c], s[c + 1]), make_float2(c2, c2),
                                        make_float2(neg_m, neg_m));
            float p0, p1;
            if (poly_pair(i)) {
                const float2 e = exp2_poly2(x);
                p0 = e.x;
                p1 = e.y;
            } else {
                p0 = ptx::ex2(x.x);
                p1 = ptx::ex2(x.y);
            }
            if (kPartial) {
                p0 = c < valid ? p0 : 0.f;
                p1 = c + 1 < valid ? p1 : 0.f;
            }
            pk[i] = ptx::pack2<false>(p0, p1);
            if (i & 1) acc1 = ptx::fadd2(acc1, make_float2(p0, p1));
            else acc0 = ptx::fadd2(acc0, make_float2(p0, p1));
        }
        ptx::tmem_st16(tP + 16 * q, pk);
    }
    return (acc0.x + acc0.y) + (acc1.x + acc1.y);
}

// One V block (a 128 x DP tile, 16-bit elements, any swizzle: the conversion
// is elementwise and in place) from bf16 to f16, by the 64 threads of the two
// converter warps; ct is the thread's index among them.  Returns the largest
// |v| seen, so that values outside f16's range can be reported.
template <int TILE>
__device__ __forceinline__ float convert_v_tile(uint8_t* tile, int ct, float vmax) {
    constexpr int NV = TILE / 16 / 64;  // 16-byte vectors per thread
    static_assert(TILE % (16 * 64) == 0, "converter split");
    uint4* const v = reinterpret_cast<uint4*>(tile);
#pragma unroll 4
    for (int i = 0; i < NV; ++i) {
        uint4 w = v[ct + 64 * i];
        uint32_t* const u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(u[e] << 16);
            const float hi = __uint_as_float(u[e] & 0xFFFF0000u);
            vmax = ptx::fmax3(vmax, fabsf(lo), fabsf(hi));
            u[e] = ptx::pack2<false>(lo, hi);
        }
        v[ct + 64 * i] = w;
    }
    return vmax;
}

// Multiply this thread's row of O (DP columns of TMEM at tO) by alpha.
template <int DP>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll
    for (int c = 0; c + 32 <= DP; c += 32) {
        uint32_t r[32];
        ptx::tmem_ld32(tO + c, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
        ptx::tmem_st32(tO + c, r);
    }
    if (DP % 32) {
        constexpr int c = DP - 16;
        uint32_t r[16];
        ptx::tmem_ld16(tO + c, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
        ptx::tmem_st16(tO + c, r);
    }
}

// O / l for this thread's row, converted and stored with 16-byte stores.  All
// DP columns are read out of TMEM first; then, if o_empty is nonzero, that
// barrier is told that O may be overwritten (the next item's first P.V waits
// for it) before the conversion and the global stores, which need only
// registers.
template <int DP, bool kBF16>
__device__ __forceinline__ void store_row(uint32_t tO, float inv_l, uint8_t* orow, bool row_ok, int D,
                                          uint32_t o_empty) {
    constexpr int NF = DP / 32;
    constexpr bool kTail = DP % 32 != 0;
    uint32_t r[NF > 0 ? NF : 1][32];
    uint32_t rt[16];
#pragma unroll
    for (int c = 0; c < NF; ++c) ptx::tmem_ld32(tO + 32 * c, r[c]);
    if (kTail) ptx::tmem_ld16(tO + DP - 16, rt);
    ptx::tmem_wait_ld();
    if (o_empty != 0u) {
        ptx::tc_fence_before();
        ptx::mbar_arrive(o_empty);
    }
    auto col_word = [&](int col) -> float {  // column col of O (compile-time index after unrolling)
        return __uint_as_float(col < 32 * NF ? r[col >> 5][col & 31] : rt[col - (DP - 16)]);
    };
#pragma unroll
    for (int col = 0; col < DP; col += 8) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = ptx::pack2<kBF16>(col_word(col + 2 * i) * inv_l, col_word(col + 2 * i + 1) * inv_l);
        if (row_ok && col + 8 <= D) ptx::st_global_v4(orow + 2 * col, w[0], w[1], w[2], w[3]);
    }
}

// The merged row of a split item, f0 * O_0 + f1 * O_1 (the weights carry the
// two halves' rescale to the common maximum and the 1 / l), converted and
// stored; 32 columns of each half at a time.
template <int DP, bool kBF16>
__device__ __forceinline__ void store_row_merged(uint32_t tO0, uint32_t tO1, float f0, float f1, uint8_t* orow,
                                                 bool row_ok, int D) {
    auto emit = [&](int col, const uint32_t* a, const uint32_t* b, int n) {
        for (int g = 0; g < n / 8; ++g) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int x = 8 * g + 2 * i;
                w[i] = ptx::pack2<kBF16>(fmaf(__uint_as_float(a[x]), f0, __uint_as_float(b[x]) * f1),
                                         fmaf(__uint_as_float(a[x + 1]), f0, __uint_as_float(b[x + 1]) * f1));
            }
            if (row_ok && col + 8 * g + 8 <= D) ptx::st_global_v4(orow + 2 * (col + 8 * g), w[0], w[1], w[2], w[3]);
        }
    };
#pragma unroll
    for (int c = 0; c + 32 <= DP; c += 32) {
        uint32_t a[32], b[32];
        ptx::tmem_ld32(tO0 + c, a);
        ptx::tmem_ld32(tO1 + c, b);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 4; ++g) emit(c + 8 * g, a + 8 * g, b + 8 * g, 8);
    }
    if (DP % 32) {
        constexpr int c = DP - 16;
        uint32_t a[16], b[16];
        ptx::tmem_ld16(tO0 + c, a);
        ptx::tmem_ld16(tO1 + c, b);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 2; ++g) emit(c + 8 * g, a + 8 * g, b + 8 * g, 8);
    }
}

// Zeros for this thread's output row (a query that sees no key).
__device__ __forceinline__ void store_zero_row(uint8_t* orow, bool row_ok, int D) {
    if (!row_ok) return;
    for (int col = 0; col + 8 <= D; col += 8) ptx::st_global_v4(orow + 2 * col, 0u, 0u, 0u, 0u);
}

// ---------------------------------------------------------------- work items

// A work item: (b, h, group of query tiles) -- for a ragged batch (segment,
// h, group).  It attends over the n query rows starting at token tok0 + q0
// of batch b and the nk keys starting at token tok0.
struct Item {
    int b, h, q0, nt, tok0, n, nk;  // n query rows, nk keys (equal except for cross lengths)
};

// Item i.  Items are numbered so that those of one (b, h) are adjacent and
// the CTAs running at once share K/V in L2.
template <bool kVarlen>
__device__ __forceinline__ Item item_of(const FwdParams& p, const SegTable<kVarlen>& seg, int i) {
    Item it;
    int qg;
    if constexpr (kVarlen) {
        // the segment whose items contain i: the last s with item0[s] <= i
        // (an empty segment has no items, so it is never the answer)
        int lo = 0, hi = seg.n;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (seg.item0[mid] <= i) lo = mid;
            else hi = mid;
        }
        const int local = i - seg.item0[lo];
        it.h = local / seg.qgroups[lo];
        qg = local - it.h * seg.qgroups[lo];
        it.b = 0;
        it.tok0 = seg.start[lo];
        it.n = seg.len[lo];
        it.nk = it.n;
    } else {
        qg = i % p.n_qgroups;
        // with the causal mask a later query group sees more keys: take each
        // head's longest group first, so the grid's last CTAs are short ones
        if (p.causal) qg = p.n_qgroups - 1 - qg;
        const int bh = i / p.n_qgroups;
        it.h = bh % p.H;
        it.b = bh / p.H;
        it.tok0 = 0;
        it.n = p.N;
        it.nk = p.Nk;
    }
    it.q0 = qg * (p.tiles_per_cta * kTileRows);
    it.nt = (p.split || (p.tiles_per_cta == 2 && it.q0 + kTileRows < it.n)) ? 2 : 1;
    return it;
}

// The CTA's k-th work item: looping CTAs take items blockIdx.x + k * gridDim.x.
__device__ __forceinline__ int local_item(int k) { return (int)blockIdx.x + k * (int)gridDim.x; }

// Key blocks each tile of an item runs over: its keys, and with the causal
// mask only up to the last key its last query row sees (0 if no row sees any
// key).  A split item's two halves take ceil(blocks / 2) each (the upper half
// starts at that block; with an odd count its last block lies past the keys
// and is masked whole).
__device__ __forceinline__ int item_kblocks(const FwdParams& p, const Item& it) {
    int keys = it.nk;
    if (p.causal) keys = max(0, min(keys, min(it.q0 + it.nt * kTileRows, it.n) + p.causal_off));
    const int blocks = (keys + kBlockKeys - 1) / kBlockKeys;
    return p.split ? (blocks + 1) / 2 : blocks;
}

// ---------------------------------------------------------------- roles

// The TMA producer (one lane): for each of the CTA's items its T Q tiles
// (Q buffer k % NQ, refilled once the S products of item k - NQ have read
// it), then K_j and V_j of each key block into ring entries 2g and 2g + 1
// (slot = entry % kStages, refilled once the MMAs that read the previous
// occupant have completed).  Before returning it waits (bounded) for every
// copy it started, so that no copy lands after an abort has ended the CTA.
// Every item of the CTA has nkb key blocks per tile.  kSplit: both tiles are
// the item's one query tile (its Q is loaded into both buffers), tile t runs
// over key blocks t*nkb + j, and every unit has its own K/V pair: the ring
// takes K_j, V_j, K_{nkb+j}, V_{nkb+j} for each j.
template <int DP, int NQ, int kStages, bool kLoop, bool kVarlen, bool kSplit = false>
__device__ __forceinline__ void produce(const FwdParams& p, const SegTable<kVarlen>& seg, uint32_t sQ, uint32_t sKV,
                                        uint32_t sBar, volatile int* abort_flag, int n_my, int T, int nkb,
                                        uint64_t tmo) {
    constexpr int TILE = tile_bytes(DP);
    constexpr int NCH = chunk_count(DP);
    auto bar = [&](int i) -> uint32_t { return sBar + 8u * (uint32_t)i; };
#pragma unroll
    for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int m = 0; m < 3; ++m) ptx::prefetch_tensormap(&p.maps[m][width_class(chunk_width(DP, c))]);
    int r = 0;  // K/V ring entries issued so far (K_j, V_j of each item in turn)
    // last item whose Q tile 0 / tile 1 was issued (two scalars rather than an
    // array indexed by the tile, which would live in local memory)
    int q_last0 = -1, q_last1 = -1;
    bool ok = true;
    for (int k = 0; k < n_my && ok; ++k) {
        const Item it = item_of<kVarlen>(p, seg, local_item(k));
        const int qb = k % NQ;
        for (int t = 0; t < T && ok; ++t) {
            // Q buffer qb of tile t was last read by the S products of item k - NQ
            if (kLoop && k >= NQ &&
                !wait_one(bar(kBarQEmpty + 2 * qb + t), (uint32_t)((k / NQ) - 1) & 1u, abort_flag, tmo, 12)) {
                ok = false;
                break;
            }
            ptx::mbar_arrive_expect_tx(bar(kBarQFull + 2 * qb + t), TILE);
#pragma unroll
            for (int c = 0; c < NCH; ++c)
                ptx::tma_load_4d(sQ + (qb * kTilesPerCta + t) * TILE + 256 * chunk_col(DP, c),
                                 &p.maps[0][width_class(chunk_width(DP, c))], chunk_col(DP, c), it.h,
                                 it.tok0 + it.q0 + (kSplit ? 0 : t * kTileRows), it.b, bar(kBarQFull + 2 * qb + t));
            if (t == 0) q_last0 = k;
            else q_last1 = k;
        }

        for (int u = 0; u < nkb * (kSplit ? T : 1) && ok; ++u) {
            const int j = kSplit ? (u >> 1) + (u & 1) * nkb : u;  // key block of this K/V pair
            for (int kv = 0; kv < 2; ++kv, ++r) {
                const int slot = r % kStages;
                const uint32_t phase = (uint32_t)(r / kStages) & 1u;
                if (!wait_one(bar(kBarKvEmpty + slot), phase ^ 1u, abort_flag, tmo, 1)) {
                    ok = false;
                    break;
                }
                if (r == 1 && (p.flags & kFlagSkipFirstVLoad)) continue;  // test-only
                ptx::mbar_arrive_expect_tx(bar(kBarKvFull + slot), TILE);
#pragma unroll
                for (int c = 0; c < NCH; ++c)
                    ptx::tma_load_4d(sKV + slot * TILE + 256 * chunk_col(DP, c),
                                     &p.maps[1 + kv][width_class(chunk_width(DP, c))], chunk_col(DP, c),
                                     it.h / p.kv_group, it.tok0 + j * kBlockKeys, it.b, bar(kBarKvFull + slot));
            }
        }
    }
    // let every copy this CTA started land before the CTA exits (in a normal
    // run they all have; after an abort some may not have been waited for).
    // The last fill of each buffer or slot is its latest phase, so its parity
    // is unambiguous whether or not it was consumed.
    const uint64_t drain_ns = 200000000ull;
    for (int t = 0; t < T; ++t) {
        const int q_last = t == 0 ? q_last0 : q_last1;
        for (int k = q_last; k >= 0 && k > q_last - NQ; --k)
            wait_drain(bar(kBarQFull + 2 * (k % NQ) + t), (uint32_t)(k / NQ) & 1u, drain_ns);
    }
    for (int idx = r - 1; idx >= 0 && idx >= r - kStages; --idx) {
        if ((p.flags & kFlagSkipFirstVLoad) && idx == 1) continue;
        wait_drain(bar(kBarKvFull + idx % kStages), (uint32_t)(idx / kStages) & 1u, drain_ns);
    }
}

// The bf16 V converter (the 64 threads of two warps, ct = 0..63): V_g (ring
// entry 2g + 1) is converted to f16 in place once it lands, made visible to
// the tensor core's (async) proxy, and announced on v_ready[g % (kStages/2)]
// (64 arrivals).  The converter can run at most kStages/2 blocks ahead: V_g's
// slot is refilled only after the last P.V of the block it held.
template <int TILE, int kStages>
__device__ __forceinline__ void convert_v_blocks(uint8_t* kv_tiles, uint32_t sBar, int bar_v_ready,
                                                 volatile int* abort_flag, int nblocks, uint64_t tmo, int ct) {
    constexpr int kVSlots = kStages / 2;
    float vmax = 0.f;
    for (int g = 0; g < nblocks; ++g) {
        const int idx = 2 * g + 1;
        const int slot = idx % kStages;
        if (!wait_warp(sBar + 8u * (uint32_t)(kBarKvFull + slot), (uint32_t)(idx / kStages) & 1u, abort_flag, tmo, 14))
            break;
        vmax = convert_v_tile<TILE>(kv_tiles + slot * TILE, ct, vmax);
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(sBar + 8u * (uint32_t)(bar_v_ready + g % kVSlots));
    }
    if (vmax >= 65536.f) atomicOr(&g_vitattn_range, 1u);
}

// S = Q K^T for one 128 x 128 block (M = 128 query rows, N = 128 keys, K =
// DP in steps of 16), f32 into TMEM columns [d, d + 128).  Descriptors are
// built once per column chunk; a K step only adds a constant to the start
// address field (16-byte units), so the issuing thread spends its time
// issuing MMAs.
template <int DP, bool kBF16>
__device__ __forceinline__ void issue_qk(uint32_t d, uint32_t q_tile, uint32_t k_tile, uint32_t leader) {
    constexpr int NCH = chunk_count(DP);
    constexpr uint32_t idS = idesc_f16(kBF16, kBlockKeys, false);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int w = chunk_width(DP, c);
        const uint64_t qd = sdesc(q_tile + 256 * chunk_col(DP, c), 16, 16u * (uint32_t)w, swizzle_code(w));
        const uint64_t kd = sdesc(k_tile + 256 * chunk_col(DP, c), 16, 16u * (uint32_t)w, swizzle_code(w));
#pragma unroll
        for (int kk = 0; kk < w / 16; ++kk)
            ptx::mma_ss_w(d, qd + 2u * kk, kd + 2u * kk, idS, (c == 0 && kk == 0) ? 0u : 1u, leader);
    }
}

// O (+)= P V for one key block (f16 x f16): A = P, 16-bit pairs in TMEM
// columns [a, a + 64); B = the V tile (MN-major); D = O in TMEM columns
// [d, d + DP).  The 64-column chunks of V form one MMA with N = 64 * n64 (the
// second 64-column swizzle atom sits one chunk, 16 KB, further: the leading
// byte offset); narrower tail chunks get an MMA each.
template <int DP>
__device__ __forceinline__ void issue_pv(uint32_t d, uint32_t a, uint32_t v_tile, bool accumulate,
                                         uint32_t leader) {
    constexpr int NCH = chunk_count(DP);
    constexpr int N64 = DP / 64;
    constexpr int NTAIL = NCH - N64;
    const uint64_t vd64 = sdesc(v_tile, 128u * 128u, 16u * 64u, swizzle_code(64));
    uint64_t vdt[NTAIL > 0 ? NTAIL : 1];
#pragma unroll
    for (int i = 0; i < NTAIL; ++i) {
        const int c = N64 + i;
        const int w = chunk_width(DP, c);
        vdt[i] = sdesc(v_tile + 256 * chunk_col(DP, c), 256u * (uint32_t)w, 16u * (uint32_t)w, swizzle_code(w));
    }
#pragma unroll
    for (int ks = 0; ks < kBlockKeys / 16; ++ks) {
        const uint32_t acc = (accumulate || ks > 0) ? 1u : 0u;
        if (N64 > 0)
            ptx::mma_ts_w(d, a + (uint32_t)(ks * 8), vd64 + (uint64_t)(2 * 64 * ks), idesc_f16(false, 64 * N64, true),
                          acc, leader);
#pragma unroll
        for (int i = 0; i < NTAIL; ++i) {
            const int c = N64 + i;
            const int w = chunk_width(DP, c);
            ptx::mma_ts_w(d + (uint32_t)chunk_col(DP, c), a + (uint32_t)(ks * 8), vdt[i] + (uint64_t)(2 * w * ks),
                          idesc_f16(false, w, true), acc, leader);
        }
    }
}

// ---------------------------------------------------------------- the kernel

// kLoop: the CTA loops over work items (grid smaller than the item count);
// without it every CTA owns exactly one item and the item loops fold away.
// kVarlen: a ragged batch (tokens of several images packed along the N axis
// of a B = 1 tensor, described by `seg`); each work item attends within its
// own segment.  Ragged batches run one item per CTA.
// kSplit (one item per CTA): the item is one query tile, and the two softmax
// warpgroups take the lower and upper halves of its key blocks with their
// own running (m, l, O); at the end the upper half hands (m, l) over shared
// memory to the lower, which reads the upper O out of TMEM and writes
//   O = (O_0 2^(m_0 - m) + O_1 2^(m_1 - m)) / (l_0 2^(m_0 - m) + l_1 2^(m_1 - m)),
// m = max(m_0, m_1): the same online-softmax merge the key blocks of one half
// already go through, applied once more.  This halves the serial chain of a
// CTA when the items are too few to fill the SMs with two tiles each.
template <int DP, bool kBF16, bool kLoop, bool kVarlen, bool kSplit = false>
__global__ void __launch_bounds__(kThreads, 1) fwd_kernel(const __grid_constant__ FwdParams p,
                                                          const __grid_constant__ SegTable<kVarlen> seg) {
    constexpr int TILE = tile_bytes(DP);
    constexpr int NCH = chunk_count(DP);
    static_assert(DP % 16 == 0 && DP >= 16 && DP <= 128, "head dim padding");
    static_assert(!(kLoop && kVarlen), "ragged batches run one work item per CTA");
    static_assert(!kSplit || (!kLoop && !kVarlen), "split items run one per CTA, dense layout");

    constexpr int NQ = q_buffers(DP, kLoop);
    constexpr int kStages = kv_stages(DP, kSplit);
    constexpr int kVSlots = kStages / 2;  // V_g sits in V slot g % kVSlots, its use g / kVSlots
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    const uint32_t sQ = base;  // [NQ][2 tiles]
    const uint32_t sKV = base + NQ * kTilesPerCta * TILE;
    const uint32_t sBar = base + (NQ * kTilesPerCta + kStages) * TILE;
    uint32_t* const tmem_holder =
        reinterpret_cast<uint32_t*>(base_ptr + (NQ * kTilesPerCta + kStages) * TILE + kNumBars * 8);
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    float* const merge_ml = reinterpret_cast<float*>(tmem_holder + 4);  // [2][128] (m, l) of the upper half
    auto bar = [&](int i) -> uint32_t { return sBar + 8u * (uint32_t)i; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // This CTA's k-th item is local_item(k).  The host launches fewer CTAs
    // than items only when every item has the same number of query tiles (T
    // below) and of key blocks (nkb: the causal mask runs one CTA per item).
    auto my_item = [&](int k) -> Item { return item_of<kVarlen>(p, seg, local_item(k)); };
    const int n_my = kLoop ? (p.n_items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 1;
    const Item first = my_item(0);
    const int T = first.nt;
    // key blocks of this CTA's items; with the causal mask, only up to the last
    // key the item's last query row sees (0 if no row sees any key)
    const int nkb = kLoop ? p.n_kblocks : item_kblocks(p, first);
    const uint64_t tmo = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 * kMaxQBufs; ++i) {
            ptx::mbar_init(bar(kBarQFull + i), 1);
            ptx::mbar_init(bar(kBarQEmpty + i), 1);
        }
        for (int s = 0; s < kMaxStages; ++s) {
            ptx::mbar_init(bar(kBarKvFull + s), 1);
            ptx::mbar_init(bar(kBarKvEmpty + s), 1);
        }
        for (int b = 0; b < kMaxSBufs; ++b) ptx::mbar_init(bar(kBarSFull + b), 1);
        for (int t = 0; t < 2; ++t) {
            ptx::mbar_init(bar(kBarPFull + 2 * t), 4 * 32);
            ptx::mbar_init(bar(kBarPFull + 2 * t + 1), 4 * 32);
            ptx::mbar_init(bar(kBarOReady + t), 1);
            ptx::mbar_init(bar(kBarOFull + t), 1);
            ptx::mbar_init(bar(kBarOEmpty + t), 4 * 32);
            for (int vs = t; vs < kMaxStages / 2; vs += 2) ptx::mbar_init(bar(kBarVReady + vs), 2 * 32);
        }
        ptx::mbar_init(bar(kBarDrain), 1);
        ptx::mbar_init(bar(kBarMerge), 4 * 32);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kLoadWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_holder), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    // Each role's register budget is set inside its own branch, so that the
    // compiler allocates the softmax code against the larger budget.
    if (warp >= kLoadWarp) {
    ptx::setmaxnreg_dec<kSideRegs>();
    if (warp == kLoadWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0)
            produce<DP, NQ, kStages, kLoop, kVarlen, kSplit>(p, seg, sQ, sKV, sBar, abort_flag, n_my, T, nkb, tmo);
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the issue loop (its control flow and descriptors
        // stay warp-uniform); one elected lane issues each MMA and commit.
        {
            const uint32_t leader = ptx::elect_one();
            constexpr int NS = s_buffers(DP);
            constexpr int OC = o_cols(DP);
            auto mma_s = [&](int qtile, int slot, int buf) {
                issue_qk<DP, kBF16>(tmem + (uint32_t)(buf * kBlockKeys), sQ + qtile * TILE, sKV + slot * TILE, leader);
            };
            auto mma_pv = [&](int t, int slot, int buf, bool accumulate) {
                issue_pv<DP>(tmem + (uint32_t)(NS * kBlockKeys + t * OC), tmem + (uint32_t)(buf * kBlockKeys),
                             sKV + slot * TILE, accumulate, leader);
            };
            // K_j and V_j occupy ring entries 2j and 2j+1 (the producer's order).
            auto kv_slot = [](int idx) { return idx % kStages; };
            auto kv_parity = [](int idx) { return (uint32_t)(idx / kStages) & 1u; };
            const int total = n_my * T * nkb;  // units of all this CTA's items
            const int ns = active_s_buffers(NS, T);
            const bool track_pv = pv_done_needed(ns, T);
            // A cursor walks the units s = T*j + t in order, keeping (t, j) and the
            // S buffer s mod ns without divisions (this thread is on the critical path).
            struct Cursor {
                int t, j, k, g, buf;  // tile, block, item (local index), block count g = k*nkb + j, S buffer
            };
            // The K/V pair a unit reads: block g's, shared by its tiles -- or, for a
            // split item, the unit's own (its tiles read different key blocks).
            auto kv_pair = [&](const Cursor& c) -> int { return kSplit ? T * c.g + c.t : c.g; };
            auto advance = [&](Cursor& c) {
                if (++c.t == T) {
                    c.t = 0;
                    ++c.g;
                    if (++c.j == nkb) {
                        c.j = 0;
                        ++c.k;
                    }
                }
                if (++c.buf == ns) c.buf = 0;
            };
            // S for one unit into its buffer; K_j is waited for by its first unit
            // and released after its last.
            auto issue_s = [&](const Cursor& c) -> bool {
                const int qb = c.k % NQ;
                if (c.j == 0) {  // first S of this tile in this item: its Q tile
                    if (!wait_warp(bar(kBarQFull + 2 * qb + c.t), (uint32_t)(c.k / NQ) & 1u, abort_flag, tmo, 2))
                        return false;
                    ptx::tc_fence_after();
                }
                const int e = kv_pair(c);
                if (kSplit || c.t == 0) {
                    if (!wait_warp(bar(kBarKvFull + kv_slot(2 * e)), kv_parity(2 * e), abort_flag, tmo, 3))
                        return false;
                    ptx::tc_fence_after();
                }
                mma_s(qb * kTilesPerCta + c.t, kv_slot(2 * e), c.buf);
                ptx::mma_commit_w(bar(kBarSFull + c.buf), leader);
                if (kSplit || c.t == T - 1) ptx::mma_commit_w(bar(kBarKvEmpty + kv_slot(2 * e)), leader);
                if (kLoop && c.j == nkb - 1) ptx::mma_commit_w(bar(kBarQEmpty + 2 * qb + c.t), leader);
                return true;
            };
            // O_t += P V_j; V_j is waited for by its first unit (landed, and for
            // bf16 inputs converted to f16) and released after its last.  V-ready
            // is per V slot: the converter reaches the slot's next block only after
            // it lands there, which needs the last P.V of this one, so the parity is
            // unambiguous.  (K/V pair e: K in ring entry 2e, V in 2e + 1.)
            auto issue_pv = [&](const Cursor& c) -> bool {
                const int t = c.t, j = c.j, g = c.g;
                const int e = kv_pair(c);
                if ((kSplit || t == 0) &&
                    !(kBF16 ? wait_warp(bar(kBarVReady + e % kVSlots), (uint32_t)(e / kVSlots) & 1u, abort_flag,
                                        tmo, 4)
                            : wait_warp(bar(kBarKvFull + kv_slot(2 * e + 1)), kv_parity(2 * e + 1), abort_flag,
                                       tmo, 4)))
                    return false;
                // the first product of an item overwrites O_t: the previous item's
                // epilogue must have read it out
                if (kLoop && j == 0 && c.k > 0 &&
                    !wait_warp(bar(kBarOEmpty + t), (uint32_t)(c.k - 1) & 1u, abort_flag, tmo, 13))
                    return false;
                if (!wait_warp(bar(kBarPFull + 2 * t + (g & 1)), (uint32_t)(g >> 1) & 1u, abort_flag, tmo, 5))
                    return false;
                ptx::tc_fence_after();
                mma_pv(t, kv_slot(2 * e + 1), c.buf, j > 0);
                if (track_pv) ptx::mma_commit_w(bar(kBarOReady + t), leader);
                if (kSplit || t == T - 1) ptx::mma_commit_w(bar(kBarKvEmpty + kv_slot(2 * e + 1)), leader);
                if (j == nkb - 1) ptx::mma_commit_w(bar(kBarOFull + t), leader);
                return true;
            };

            bool ok = true;
            Cursor cs{0, 0, 0, 0, 0};  // next unit whose S is issued
            Cursor cp{0, 0, 0, 0, 0};  // next unit whose P.V is issued
            int issued_s = 0;
            for (; issued_s < ns && issued_s < total && ok; ++issued_s) {
                ok = issue_s(cs);
                advance(cs);
            }
            for (int s = 0; s < total && ok; ++s) {
                ok = issue_pv(cp);
                advance(cp);
                if (ok && issued_s < total) {
                    ok = issue_s(cs);
                    advance(cs);
                    ++issued_s;
                }
            }
            if (!ok) {
                // every MMA issued so far must finish before TMEM is freed
                ptx::mma_commit_w(bar(kBarDrain), leader);
                wait_drain(bar(kBarDrain), 0, 200000000ull);
            }
        }
        __syncwarp();
    } else if (kBF16) {
        // ------------------------------------------------------------ V converter (bf16)
        convert_v_blocks<TILE, kStages>(base_ptr + (sKV - base), sBar, kBarVReady, abort_flag,
                                        n_my * nkb * (kSplit ? T : 1), tmo, (int)threadIdx.x - kConvWarp * 32);
    }
    } else {
        ptx::setmaxnreg_inc<kSoftmaxRegs>();
        // ------------------------------------------------------------ softmax
        const int t = warp >> 2;
        const int wq = warp & 3;
        if (t < T) {
            constexpr int NS = s_buffers(DP);
            const int ns = active_s_buffers(NS, T);
            const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
            const uint32_t tO = tmem + lane_base + (uint32_t)(NS * kBlockKeys + t * o_cols(DP));
            const float c2 = p.scale_log2;
            const bool neg = c2 < 0.f;
            bool ok = true;
            // unit = T*g + t (g = blocks of this tile so far, over all items) lives
            // in S buffer unit % ns, as phase unit / ns of that buffer's barrier;
            // both advance by T units per block.
            int sbuf = t % ns, sphase = t / ns;
            int g = 0;
            int o_phase = 0;  // items so far whose O_t has been (or is being) accumulated
            // The epilogue of item k (wait for its last P.V, read O_t out, store
            // O / l) runs after the first block of item k + 1 has been handed to
            // the MMA warp, so that the last P.V's latency is hidden behind that
            // block's softmax; O_t is released before the global stores.
            auto finish = [&](int k, float m_used, float l, int kb, int phase) -> bool {
                if (kb > 0 && !wait_warp(bar(kBarOFull + t), (uint32_t)phase & 1u, abort_flag, tmo, 8)) return false;
                ptx::tc_fence_after();
                const Item it = my_item(k);
                const int row = it.q0 + (kSplit ? 0 : t * kTileRows) + wq * 32 + lane;
                uint8_t* orow = reinterpret_cast<uint8_t*>(p.out) +
                                (((size_t)it.b * p.N + (size_t)it.tok0 + (size_t)min(row, it.n - 1)) *
                                     (size_t)p.out_ts + (size_t)it.h * p.D) * 2;
                const uint32_t o_empty = kLoop ? bar(kBarOEmpty + t) : 0u;
                if constexpr (kSplit) {
                    // the upper half hands its (m, l) over; the lower half waits for
                    // both halves' last P.V and that hand-over, then merges
                    const int rl = wq * 32 + lane;
                    if (t == 1) {
                        merge_ml[rl] = m_used;
                        merge_ml[kTileRows + rl] = l;
                        ptx::mbar_arrive(bar(kBarMerge));
                        return true;
                    }
                    if (!wait_warp(bar(kBarOFull + 1), 0u, abort_flag, tmo, 15) ||
                        !wait_warp(bar(kBarMerge), 0u, abort_flag, tmo, 16))
                        return false;
                    ptx::tc_fence_after();
                    const float m1 = merge_ml[rl], l1 = merge_ml[kTileRows + rl];
                    const float m = fmaxf(m_used, m1);
                    const float a0 = m_used == -INFINITY ? 0.f : ptx::ex2(m_used - m);
                    const float a1 = m1 == -INFINITY ? 0.f : ptx::ex2(m1 - m);
                    const float lm = l * a0 + l1 * a1;
                    const float inv = lm > 0.f ? 1.f / lm : 0.f;
                    store_row_merged<DP, kBF16>(tO, tO + (uint32_t)o_cols(DP), a0 * inv, a1 * inv, orow, row < it.n,
                                                p.D);
                    if (p.lse != nullptr && row < it.n)
                        p.lse[((size_t)it.b * p.H + it.h) * p.N + it.tok0 + row] =
                            lm > 0.f ? (m + log2f(lm)) * 0.6931471805599453f : -INFINITY;
                    return true;
                }
                // a row that saw no key (causal, more queries than keys) is 0
                if (kb > 0) {
                    store_row<DP, kBF16>(tO, l > 0.f ? 1.f / l : 0.f, orow, row < it.n, p.D, o_empty);
                } else {
                    store_zero_row(orow, row < it.n, p.D);
                    if (kLoop) ptx::mbar_arrive(o_empty);
                }
                if (p.lse != nullptr && row < it.n)
                    p.lse[((size_t)it.b * p.H + it.h) * p.N + it.tok0 + row] =
                        l > 0.f ? (m_used + log2f(l)) * 0.6931471805599453f : -INFINITY;
                return true;
            };
            // the item whose epilogue is pending (-1: none) and its row state
            int pend = -1, pend_kb = 0, pend_phase = 0;
            float pend_m = 0.f, pend_l = 0.f;
            for (int k = 0; k < n_my && ok; ++k) {
            const Item it = my_item(k);
            const int kb = nkb;
            const int row = it.q0 + (kSplit ? 0 : t * kTileRows) + wq * 32 + lane;
            const int kb0 = kSplit ? t * kb : 0;  // this tile's first key block
            float m_used = -INFINITY;
            float l = 0.f;
            for (int j = 0; j < kb; ++j, ++g) {
                const uint32_t tS = tmem + lane_base + (uint32_t)(sbuf * kBlockKeys);
                const uint32_t s_bar = bar(kBarSFull + sbuf);
                const uint32_t s_par = (uint32_t)sphase & 1u;
                sbuf += T;
                if (sbuf >= ns) {
                    sbuf -= ns;
                    ++sphase;
                }
                if (!wait_warp(s_bar, s_par, abort_flag, tmo, 7)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                float s[kBlockKeys];
                {
                    uint32_t r[4][32];
#pragma unroll
                    for (int q = 0; q < 4; ++q) ptx::tmem_ld32(tS + 32 * q, r[q]);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 4; ++q)
#pragma unroll
                        for (int i = 0; i < 32; ++i) s[32 * q + i] = __uint_as_float(r[q][i]);
                }
                // keys of this block the row sees: the ragged tail, and with the
                // causal mask the row's own limit (<= 0: none); "partial" is decided
                // warp-wide because the exp path holds warp-collective TMEM stores
                int valid = min(kBlockKeys, it.nk - (kb0 + j) * kBlockKeys);
                if (p.causal) valid = min(valid, row + p.causal_off + 1 - (kb0 + j) * kBlockKeys);
                const bool partial = __any_sync(0xffffffffu, valid < kBlockKeys);
                const float ext = partial ? (neg ? row_extreme<true, true>(s, valid)
                                                 : row_extreme<true, false>(s, valid))
                                          : (neg ? row_extreme<false, true>(s, valid)
                                                 : row_extreme<false, false>(s, valid));
                const float m_blk = valid > 0 ? ext * c2 : -INFINITY;
                const float m_new = fmaxf(m_used, m_blk);
                const bool need = (m_new - m_used) > kRescaleThreshold;
                float alpha = 1.f;
                if (need) {
                    alpha = ptx::ex2(m_used - m_new);
                    m_used = m_new;
                    l *= alpha;
                }
                l += partial ? exp_pack_store<true>(s, valid, c2, -m_used, tS)
                             : exp_pack_store<false>(s, valid, c2, -m_used, tS);
                // Bring O_t (P.V up to block j-1) to the new reference maximum before
                // P_t,j.V_j is issued.  The product of block j-1 may still be running:
                // wait for it (phase j-1 of the per-tile "P.V done" barrier; the phase
                // of block j-2 has completed by now, so the parity is unambiguous).
                if (j > 0 && __any_sync(0xffffffffu, need)) {
                    if (pv_done_needed(ns, T) &&
                        !wait_warp(bar(kBarOReady + t), (uint32_t)(g - 1) & 1u, abort_flag, tmo, 11)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    rescale_o<DP>(tO, alpha);
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(bar(kBarPFull + 2 * t + (g & 1)));
                // the previous item's epilogue (its O_t is released before this
                // item's first P.V can start)
                if (kLoop && j == 0 && pend >= 0) {
                    ok = finish(pend, pend_m, pend_l, pend_kb, pend_phase);
                    pend = -1;
                    if (!ok) break;
                }
            }
            if (!ok) break;
            // an item without key blocks has nothing for its epilogue to wait for
            if (kLoop && pend >= 0) {
                ok = finish(pend, pend_m, pend_l, pend_kb, pend_phase);
                pend = -1;
                if (!ok) break;
            }
            pend = k;
            pend_m = m_used;
            pend_l = l;
            pend_kb = kb;
            pend_phase = o_phase;
            if (kb > 0) ++o_phase;
            }
            if (ok && pend >= 0) ok = finish(pend, pend_m, pend_l, pend_kb, pend_phase);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kLoadWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}


}  // namespace vitattn
