// fsdpk_device.cuh -- device helpers and launch geometry shared by the kernel
// files of libfsdpk.so (fsdpk_gather.cu, fsdpk_reduce.cu, fsdpk_update.cu).
// Every stage is HBM-bound streaming (well under one flop per byte), so
// nothing here uses tensor cores: 16-byte coalesced accesses, enough bytes in
// flight per SM to cover HBM latency, streaming (evict-first) cache hints for
// data touched once, one CTA per work item launched in order.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "fsdpk_internal.h"

namespace fsdpk {
namespace {

constexpr int kThreads = 256;

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) {
    return __uint_as_float(h << 16);
}

// 8 bf16 (one 16-byte vector) -> 8 fp32, exact widening.
__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
    x[0] = __uint_as_float(w.x << 16);
    x[1] = __uint_as_float(w.x & 0xFFFF0000u);
    x[2] = __uint_as_float(w.y << 16);
    x[3] = __uint_as_float(w.y & 0xFFFF0000u);
    x[4] = __uint_as_float(w.z << 16);
    x[5] = __uint_as_float(w.z & 0xFFFF0000u);
    x[6] = __uint_as_float(w.w << 16);
    x[7] = __uint_as_float(w.w & 0xFFFF0000u);
}

// Two fp32 -> one bf16x2 word (round to nearest even); lo in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// The 8 bf16 elements that start D (1..7) elements into the 16 elements a:b
// (a at the lower address): word j of the result is bits [16*D, 16*D + 32)
// of the 64-bit pair (w[j + D/2 + 1] : w[j + D/2]).
__device__ __forceinline__ uint4 shift_bf16x8(const uint4& a, const uint4& b, int D) {
    const int s = D >> 1;
    const uint32_t sh = (D & 1) ? 16u : 0u;
    const uint32_t w0 = s == 0 ? a.x : s == 1 ? a.y : s == 2 ? a.z : a.w;
    const uint32_t w1 = s == 0 ? a.y : s == 1 ? a.z : s == 2 ? a.w : b.x;
    const uint32_t w2 = s == 0 ? a.z : s == 1 ? a.w : s == 2 ? b.x : b.y;
    const uint32_t w3 = s == 0 ? a.w : s == 1 ? b.x : s == 2 ? b.y : b.z;
    const uint32_t w4 = s == 0 ? b.x : s == 1 ? b.y : s == 2 ? b.z : b.w;
    return make_uint4(__funnelshift_r(w0, w1, sh), __funnelshift_r(w1, w2, sh),
                      __funnelshift_r(w2, w3, sh), __funnelshift_r(w3, w4, sh));
}

// Aligned source vector load.  Unshifted, every vector is read once, so it
// streams past L1; shifted, the neighbouring thread reads the same vector as
// its second operand, so it is kept in L1 (read-only path).
template <bool SHIFTED>
__device__ __forceinline__ uint4 ld_src(const uint4* p) {
    if constexpr (SHIFTED) {
        return __ldg(p);
    } else {
        return __ldcs(p);
    }
}

// Elements to peel before `p` reaches a 16-byte boundary (capped at len).
template <typename T>
__device__ __forceinline__ int64_t head_to_16B(const T* p, int64_t len) {
    const int64_t h = (int64_t)((16u - (reinterpret_cast<uintptr_t>(p) & 15u)) & 15u) / sizeof(T);
    return h < len ? h : len;
}

// Position, in bf16 elements, of `p` inside its 16-byte vector.
__device__ __forceinline__ int bf16_phase(const uint16_t* p) {
    return (int)((reinterpret_cast<uintptr_t>(p) >> 1) & 7u);
}

// Zero-fill `len` fp32 elements at dst (any alignment).
__device__ __forceinline__ void zero_f32_run(float* __restrict__ dst, int64_t len) {
    int64_t head = (4 - (reinterpret_cast<uintptr_t>(dst) >> 2 & 3)) & 3;
    if (head > len) head = len;
    if (threadIdx.x < head) dst[threadIdx.x] = 0.0f;
    const int64_t nv = (len - head) >> 2;
    float4* d4 = reinterpret_cast<float4*>(dst + head);
    for (int64_t q = threadIdx.x; q < nv; q += blockDim.x)
        __stcs(d4 + q, make_float4(0.f, 0.f, 0.f, 0.f));
    const int64_t done = head + 4 * nv;
    if (threadIdx.x < len - done) dst[done + threadIdx.x] = 0.0f;
}

// Where each source rank's gradient arena starts.
//   StrideSrc: all N ranks in one buffer, rank r at base + r * stride.
//   TableSrc:  one pointer per rank (arenas in separate allocations, such as
//              peers' memory mapped into this process), held in shared memory.
// at(off) moves every rank's pointer by off elements.
struct StrideSrc {
    const uint16_t* base;
    int64_t stride;
    __device__ __forceinline__ const uint16_t* rank(int r) const { return base + r * stride; }
    __device__ __forceinline__ StrideSrc at(int64_t off) const {
        return StrideSrc{base + off, stride};
    }
};

struct TableSrc {
    const uint16_t* const* tab;
    int64_t off;
    __device__ __forceinline__ const uint16_t* rank(int r) const { return tab[r] + off; }
    __device__ __forceinline__ TableSrc at(int64_t o) const { return TableSrc{tab, off + o}; }
};

// Ranks a TableSrc kernel can address (its table lives in shared memory).
constexpr int kPeerMaxRanks = FSDP_PEER_MAX_RANKS;

// Copy an N-entry rank table into shared memory (every thread calls this).
__device__ __forceinline__ void load_rank_table(const uint16_t* const* __restrict__ g_tab,
                                                const uint16_t** s_tab, int N) {
    for (int r = threadIdx.x; r < N; r += blockDim.x) s_tab[r] = g_tab[r];
    __syncthreads();
}

template <int NR, class Src>
__device__ __forceinline__ float fold_scalar(const Src& src, int N) {
    const int n = NR ? NR : N;
    float acc = bf16_bits_to_f32(src.rank(0)[0]);
    for (int r = 1; r < n; ++r) acc = __fadd_rn(acc, bf16_bits_to_f32(src.rank(r)[0]));
    return acc;
}

// x / N in binary32, round to nearest even.  For a rank count NR known at
// compile time and a power of two, 1/NR is exact, so x * (1/NR) rounds the
// same exact value as the division, for every x (subnormal results, zeros,
// infinities and NaN included), and replaces it.
template <int NR>
__device__ __forceinline__ float div_n(float x, float fN) {
    if constexpr (NR > 0 && (NR & (NR - 1)) == 0) {
        (void)fN;
        return __fmul_rn(x, 1.0f / (float)NR);
    } else {
        return __fdiv_rn(x, fN);
    }
}

template <int NR = 0>
__device__ __forceinline__ float finish(float acc, bool avg, float fN) {
    return avg ? div_n<NR>(acc, fN) : acc;
}

__device__ __forceinline__ void store8(float* __restrict__ dst, const float (&acc)[8]) {
    float4* o = reinterpret_cast<float4*>(dst);
    __stcs(o, make_float4(acc[0], acc[1], acc[2], acc[3]));
    __stcs(o + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
}

// ---------------------------------------------------------------------------
// flat path (groups of many small parameters): one CTA per tile of the flat
// index space, kFlatV vectors of 8 elements per thread, one code per vector
// ---------------------------------------------------------------------------
constexpr int kFlatV = 4;
constexpr int64_t kFlatTile = (int64_t)kThreads * 8 * kFlatV;

// CTAs of a flat launch over `count` elements: one per tile.
inline unsigned flat_grid(int64_t count) {
    const int64_t t = (count + kFlatTile - 1) / kFlatTile;
    return (unsigned)std::min<int64_t>(std::max<int64_t>(t, 1), 0x7FFFFFFF);
}

// Elements of the mixed vectors per thread, and the CTAs that take them:
// thread t of that region has elements t + i * T (i < kFlatMixedPer; T the
// region's threads), all its loads issued together.
constexpr int kFlatMixedPer = 4;

inline int64_t flat_mixed_ctas(int64_t n_mixed) {
    return (8 * n_mixed + kThreads * kFlatMixedPer - 1) / (kThreads * kFlatMixedPer);
}

// The codes of this thread's kFlatV vectors of a flat tile (vector q0 + j *
// kThreads for j < kFlatV), read before any of them is processed; entries
// past the last vector read as mixed, which the vector loops skip.
__device__ __forceinline__ void flat_tile_codes(const int32_t* __restrict__ map, int64_t q0,
                                                int64_t nv, int32_t (&code)[kFlatV]) {
#pragma unroll
    for (int j = 0; j < kFlatV; ++j) {
        const int64_t q = q0 + (int64_t)j * kThreads;
        code[j] = q < nv ? __ldcs(map + q) : 1;
    }
}

// code[j] for a loop index j that is not unrolled (selects, no local memory).
__device__ __forceinline__ int32_t flat_pick(const int32_t (&code)[kFlatV], int j) {
    int32_t c = code[0];
#pragma unroll
    for (int t = 1; t < kFlatV; ++t)
        if (j == t) c = code[t];
    return c;
}

// Rank-ordered fold of the 8 source elements a .. a+7 of every rank (rank r
// at g + r * stride; stride a multiple of 8, so all N sources share the phase
// D of a in its 16-byte vector): aligned loads at a - D and, for D != 0, at
// a - D + 8, every rank's issued before the fold.  NR = 0: any N, ranks in
// batches of 4.
template <int NR>
__device__ __forceinline__ void flat_fold8(const uint16_t* __restrict__ g, int64_t stride, int N,
                                           int64_t a, float (&acc)[8]) {
    const int D = (int)(a & 7);
    const uint4* s = reinterpret_cast<const uint4*>(g + (a - D));
    const int64_t st4 = stride >> 3;
    if constexpr (NR != 0) {
        uint4 x[NR], y[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            x[r] = __ldg(s + r * st4);
            if (D != 0) y[r] = __ldg(s + r * st4 + 1);
            else y[r] = x[r];
        }
        unpack8(shift_bf16x8(x[0], y[0], D), acc);
#pragma unroll
        for (int r = 1; r < NR; ++r) {
            float t[8];
            unpack8(shift_bf16x8(x[r], y[r], D), t);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], t[e]);
        }
    } else {
#pragma unroll 1
        for (int r0 = 0; r0 < N; r0 += 4) {
            uint4 x[4], y[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                if (r0 + r < N) {
                    x[r] = __ldg(s + (r0 + r) * st4);
                    if (D != 0) y[r] = __ldg(s + (r0 + r) * st4 + 1);
                    else y[r] = x[r];
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                if (r0 + r < N) {
                    float t[8];
                    unpack8(shift_bf16x8(x[r], y[r], D), t);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        acc[e] = (r0 + r == 0) ? t[e] : __fadd_rn(acc[e], t[e]);
                }
            }
        }
    }
}

// One AdamW step of one element in binary32.  Where (1 - b2) * g^2 overflows
// binary32 (|g| above about 5.8e20) the stored second moment is +Inf, as the
// exact value rounds to; the update then takes sqrt(v) as
// |g| * sqrt(b2 * (v_old / g^2) + (1 - b2)), which stays finite, so the
// parameter still moves by about lr * sign(g) as AdamW's definition gives
// (rather than by 0 through m / Inf).
__device__ __forceinline__ void adamw1(float& p, float& m, float& v, float g,
                                       const AdamScalars& sc) {
    const float v_old = v;
    p = p * sc.decay;
    m = fmaf(sc.beta1, m, sc.omb1 * g);
    v = fmaf(sc.beta2, v, sc.omb2 * g * g);
    float sqrt_v = __fsqrt_rn(v);
    if (v > 3.40282347e38f && fabsf(g) <= 3.40282347e38f && v_old <= 3.40282347e38f) {
        const float a = fabsf(g);
        sqrt_v = a * __fsqrt_rn(fmaf(sc.beta2, __fdiv_rn(__fdiv_rn(v_old, a), a), sc.omb2));
    }
    const float denom = fmaf(sqrt_v, sc.inv_bc2_sqrt, sc.eps);
    p = fmaf(-sc.step_size, __fdiv_rn(m, denom), p);
}

// The AdamW scalars of step t, in binary64 on the device, in the same
// operation order as the host path.
__device__ __forceinline__ AdamScalars adam_scalars_dev(double lr, double beta1, double beta2,
                                                        double eps, double wd, int64_t t) {
    const double bc1 = 1.0 - pow(beta1, (double)t);
    const double bc2 = 1.0 - pow(beta2, (double)t);
    AdamScalars sc;
    sc.decay = (float)(1.0 - lr * wd);
    sc.beta1 = (float)beta1;
    sc.omb1 = (float)(1.0 - beta1);
    sc.beta2 = (float)beta2;
    sc.omb2 = (float)(1.0 - beta2);
    sc.step_size = (float)(lr / bc1);
    sc.inv_bc2_sqrt = (float)(1.0 / sqrt(bc2));
    sc.eps = (float)eps;
    return sc;
}

// FP8 (E4M3 "fn") helpers
// x * scale clamped to the finite E4M3 range (NaN passes through).
__device__ __forceinline__ float fp8_in(float x, float sc) {
    float y = __fmul_rn(x, sc);
    if (y > 448.0f) y = 448.0f;
    if (y < -448.0f) y = -448.0f;
    return y;
}

// Two floats -> two E4M3 bytes (lo in bits 0..7), round to nearest even.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ uint8_t e4m3(float x) {
    return (uint8_t)(e4m3x2(x, 0.0f) & 0xFFu);
}

// ---------------------------------------------------------------------------
// debug build: unit and tile checks against the extents a launch was given
// ---------------------------------------------------------------------------
#ifdef FSDPK_DEBUG
#define FSDPK_DBG_PARAM , DebugBounds dbg
#define FSDPK_DBG_ARG(x) , x
#define FSDPK_UNIT_GUARD(u, ui, what) \
    if (!unit_in_bounds(dbg, (u), (ui), (what))) continue
#define FSDPK_GUARD(ok, where) \
    if (!debug_ok(dbg, (ok), (where))) continue
#define FSDPK_THREAD_GUARD(ok, where) \
    if (!debug_ok_thread(dbg, (ok), (where))) continue
#else
#define FSDPK_DBG_PARAM
#define FSDPK_DBG_ARG(x)
#define FSDPK_UNIT_GUARD(u, ui, what) ((void)0)
#define FSDPK_GUARD(ok, where) ((void)0)
#define FSDPK_THREAD_GUARD(ok, where) ((void)0)
#endif

constexpr int kChkShard = 1;  // shard_pos + len within [0, ns)
constexpr int kChkArena = 2;  // a real unit's arena_pos + len within [0, arena)

// Every thread evaluates the same condition for a unit, so a skip is uniform
// across the block; lane 0 of each warp that sees a violation records it.
__device__ __forceinline__ bool debug_ok(const DebugBounds& b, bool ok, int64_t where) {
    if (!ok && (threadIdx.x & 31) == 0 && b.words != nullptr) {
        if (atomicAdd(b.words, 1u) == 0u) {
            b.words[1] = (uint32_t)b.kernel;
            b.words[2] = (uint32_t)where;
            b.words[3] = blockIdx.x;
        }
    }
    return ok;
}

// The flat kernels check per thread (each thread its own vectors): every
// thread that sees a violation counts it.
__device__ __forceinline__ bool debug_ok_thread(const DebugBounds& b, bool ok, int64_t where) {
    if (!ok && b.words != nullptr) {
        if (atomicAdd(b.words, 1u) == 0u) {
            b.words[1] = (uint32_t)b.kernel;
            b.words[2] = (uint32_t)where;
            b.words[3] = blockIdx.x;
        }
    }
    return ok;
}

__device__ __forceinline__ bool unit_in_bounds(const DebugBounds& b, const Unit& u, int64_t ui,
                                               int what) {
    bool ok = u.len >= 0;
    if (what & kChkShard) ok = ok && u.shard_pos >= 0 && u.shard_pos + u.len <= b.ns;
    if ((what & kChkArena) && !u.is_pad)
        ok = ok && u.arena_pos >= 0 && u.arena_pos + u.len <= b.arena;
    return debug_ok(b, ok, ui);
}

// ---------------------------------------------------------------------------
// launch geometry
// ---------------------------------------------------------------------------
// One CTA per work item (tile, unit or chunk), launched in order.  On B200 a
// grid that covers the work once streams 12-17 % faster than a persistent
// grid-stride loop with a static cyclic assignment: the hardware hands out
// CTAs in index order as slots free up, so the addresses in flight stay a
// compact window instead of drifting apart across the arrays.
inline unsigned grid_for(const fsdp_group&, const void*, int64_t items) {
    return (unsigned)std::min<int64_t>(std::max<int64_t>(items, 1), 0x7FFFFFFF);
}

}  // namespace
}  // namespace fsdpk
