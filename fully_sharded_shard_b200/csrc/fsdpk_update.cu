// fsdpk_update.cu -- the sharded AdamW update, the fused reduce-scatter +
// AdamW + next-step copy-in, and the device-side step scalars for CUDA-graph
// replay.
//   "Sharded Training: FSDP2, DTensor, Tensor and Pipeline Parallelism",
//   Fence 4 (the optimizer steps the sharded fp32 parameters, its state
//   sharded the same way) and the opening paragraph (12 bytes of fp32 state);
//   "Introduction to PyTorch FSDP2 Backend Features", Working Principle
//   (reduce-scatter, then the sharded update, then the next all-gather).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "fsdpk_device.cuh"

namespace fsdpk {
namespace {

// ---------------------------------------------------------------------------
// AdamW over the flat [N][S] buffers (pads are zero and stay zero)
// ---------------------------------------------------------------------------

constexpr int kAdamV = 2;  // float4 per array per thread
constexpr int64_t kAdamChunk4 = (int64_t)kThreads * kAdamV;  // float4 per CTA chunk

__global__ void __launch_bounds__(kThreads, 3)
k_adamw(float* __restrict__ p, float* __restrict__ m, float* __restrict__ v,
        const float* __restrict__ g, int64_t count, AdamScalars sc,
        const AdamScalars* __restrict__ sc_dev) {
    if (sc_dev != nullptr) sc = *sc_dev;  // scalars of a graph-replayed step
    const int64_t n4 = count >> 2;
    float4* p4 = reinterpret_cast<float4*>(p);
    float4* m4 = reinterpret_cast<float4*>(m);
    float4* v4 = reinterpret_cast<float4*>(v);
    const float4* g4 = reinterpret_cast<const float4*>(g);
    const int64_t n_chunks = (n4 + kAdamChunk4 - 1) / kAdamChunk4;
    for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x) {
        const int64_t q0 = c * kAdamChunk4 + threadIdx.x;
        float4 P[kAdamV], M[kAdamV], Vv[kAdamV], G[kAdamV];
#pragma unroll
        for (int k = 0; k < kAdamV; ++k) {
            const int64_t q = q0 + k * kThreads;
            if (q < n4) {
                P[k] = __ldcs(p4 + q);
                M[k] = __ldcs(m4 + q);
                Vv[k] = __ldcs(v4 + q);
                G[k] = __ldcs(g4 + q);
            }
        }
#pragma unroll
        for (int k = 0; k < kAdamV; ++k) {
            const int64_t q = q0 + k * kThreads;
            if (q < n4) {
                adamw1(P[k].x, M[k].x, Vv[k].x, G[k].x, sc);
                adamw1(P[k].y, M[k].y, Vv[k].y, G[k].y, sc);
                adamw1(P[k].z, M[k].z, Vv[k].z, G[k].z, sc);
                adamw1(P[k].w, M[k].w, Vv[k].w, G[k].w, sc);
                __stcs(p4 + q, P[k]);
                __stcs(m4 + q, M[k]);
                __stcs(v4 + q, Vv[k]);
            }
        }
    }
    // ragged tail (count % 4 elements)
    if (blockIdx.x == 0 && threadIdx.x < (count & 3)) {
        const int64_t k = 4 * n4 + threadIdx.x;
        float pp = p[k], mm = m[k], vv = v[k];
        adamw1(pp, mm, vv, g[k], sc);
        p[k] = pp;
        m[k] = mm;
        v[k] = vv;
    }
}

// ---------------------------------------------------------------------------
// fused reduce-scatter + AdamW + next-step copy-in
// For each element k of [N][S]:  g = rank-ordered fold of the N ranks'
// gradients (then / N for AVG and SUM_THEN_DIV; +0 in pad rows), AdamW on
// master/m/v[k] with g, then ag[k] = bf16_rn(master[k]) (+0 in pad rows) and
// optionally reduced[k] = g.  The fold, the division and the AdamW arithmetic
// are the ones of k_reduce_units and k_adamw, so the results are the same bits
// as the three separate stages.  The reduced gradient never goes to HBM.
// FP8 mode (delayed scaling): instead of the bf16 copy, ag8[k] =
// e4m3_rn(clamp(master[k] * scale_i, -448, 448)) with the scale of the
// previous step, and max |master| over each parameter (the next scale's amax)
// folded into amax_bits[i].
// ---------------------------------------------------------------------------

struct FusedOut {
    float* p;
    float* m;
    float* v;
    float* red;                 // may be null
    uint16_t* ag;               // bf16 next all-gather input; may be null
    uint8_t* ag8;               // FP8 mode: next all-gather input
    const float* scales;        // FP8 mode: per-parameter scale applied to ag8
    unsigned* amax_bits;        // FP8 mode: per-parameter max |updated master|
    const int32_t* unit_param;  // FP8 mode: parameter of every unit
};

// One element: adamw with g, then the optional outputs.
template <bool FP8>
__device__ __forceinline__ void fused1(const FusedOut& o, int64_t k, float g, bool pad,
                                       const AdamScalars& sc, float scale, float& mx) {
    float pp = o.p[k], mm = o.m[k], vv = o.v[k];
    adamw1(pp, mm, vv, g, sc);
    o.p[k] = pp;
    o.m[k] = mm;
    o.v[k] = vv;
    if (o.red) o.red[k] = g;
    if constexpr (FP8) {
        o.ag8[k] = pad ? (uint8_t)0 : e4m3(fp8_in(pp, scale));
        if (!pad) mx = fmaxf(mx, fabsf(pp));
    } else if (o.ag) {
        __nv_bfloat16 h = __float2bfloat16_rn(pad ? 0.0f : pp);
        o.ag[k] = *reinterpret_cast<uint16_t*>(&h);
    }
}

// Eight elements starting at an index that is a multiple of 8 (every fp32
// pointer 32-byte aligned, the bf16 pointer 16-byte and the FP8 pointer
// 8-byte aligned).
template <bool FP8>
__device__ __forceinline__ void fused8(const FusedOut& o, int64_t k, const float (&g)[8],
                                       const float4 (&P)[2], const float4 (&M)[2],
                                       const float4 (&V)[2], bool pad, const AdamScalars& sc,
                                       float scale, float& mx) {
    float pp[8] = {P[0].x, P[0].y, P[0].z, P[0].w, P[1].x, P[1].y, P[1].z, P[1].w};
    float mm[8] = {M[0].x, M[0].y, M[0].z, M[0].w, M[1].x, M[1].y, M[1].z, M[1].w};
    float vv[8] = {V[0].x, V[0].y, V[0].z, V[0].w, V[1].x, V[1].y, V[1].z, V[1].w};
#pragma unroll
    for (int e = 0; e < 8; ++e) adamw1(pp[e], mm[e], vv[e], g[e], sc);
    float4* p4 = reinterpret_cast<float4*>(o.p + k);
    float4* m4 = reinterpret_cast<float4*>(o.m + k);
    float4* v4 = reinterpret_cast<float4*>(o.v + k);
    __stcs(p4, make_float4(pp[0], pp[1], pp[2], pp[3]));
    __stcs(p4 + 1, make_float4(pp[4], pp[5], pp[6], pp[7]));
    __stcs(m4, make_float4(mm[0], mm[1], mm[2], mm[3]));
    __stcs(m4 + 1, make_float4(mm[4], mm[5], mm[6], mm[7]));
    __stcs(v4, make_float4(vv[0], vv[1], vv[2], vv[3]));
    __stcs(v4 + 1, make_float4(vv[4], vv[5], vv[6], vv[7]));
    if (o.red) store8(o.red + k, g);
    if constexpr (FP8) {
        uint2 w = make_uint2(0u, 0u);
        if (!pad) {
            uint32_t b[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                b[e] = e4m3x2(fp8_in(pp[2 * e], scale), fp8_in(pp[2 * e + 1], scale)) & 0xFFFFu;
            w = make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
#pragma unroll
            for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(pp[e]));
        }
        __stcs(reinterpret_cast<uint2*>(o.ag8 + k), w);
    } else if (o.ag) {
        uint4 w = pad ? make_uint4(0u, 0u, 0u, 0u)
                      : make_uint4(pack_bf16x2(pp[0], pp[1]), pack_bf16x2(pp[2], pp[3]),
                                   pack_bf16x2(pp[4], pp[5]), pack_bf16x2(pp[6], pp[7]));
        __stcs(reinterpret_cast<uint4*>(o.ag + k), w);
    }
}

__device__ __forceinline__ void load_pmv8(const FusedOut& o, int64_t k, float4 (&P)[2],
                                          float4 (&M)[2], float4 (&V)[2]) {
    const float4* p4 = reinterpret_cast<const float4*>(o.p + k);
    const float4* m4 = reinterpret_cast<const float4*>(o.m + k);
    const float4* v4 = reinterpret_cast<const float4*>(o.v + k);
    P[0] = __ldcs(p4);
    P[1] = __ldcs(p4 + 1);
    M[0] = __ldcs(m4);
    M[1] = __ldcs(m4 + 1);
    V[0] = __ldcs(v4);
    V[1] = __ldcs(v4 + 1);
}

// Rank-ordered fold of 8 elements; NR = N at compile time (1..8): all NR
// ranks' loads (two 16-byte vectors per rank on a misaligned run) are issued
// before the fold.  NR = 0 (any N): ranks in batches of 4.
template <int NR, bool SHIFTED, class Src>
__device__ __forceinline__ void fold8(const Src& src_al, int N, int q, int D, float (&acc)[8]) {
    if constexpr (NR != 0) {
        uint4 a[NR], b[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            const uint4* s = reinterpret_cast<const uint4*>(src_al.rank(r)) + q;
            a[r] = ld_src<SHIFTED>(s);
            if constexpr (SHIFTED) b[r] = ld_src<SHIFTED>(s + 1);
        }
        unpack8(SHIFTED ? shift_bf16x8(a[0], b[0], D) : a[0], acc);
#pragma unroll
        for (int r = 1; r < NR; ++r) {
            float x[8];
            unpack8(SHIFTED ? shift_bf16x8(a[r], b[r], D) : a[r], x);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], x[e]);
        }
    } else {
#pragma unroll 1
        for (int r0 = 0; r0 < N; r0 += 4) {
            uint4 a[4], b[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                if (r0 + r < N) {
                    const uint4* s = reinterpret_cast<const uint4*>(src_al.rank(r0 + r)) + q;
                    a[r] = ld_src<SHIFTED>(s);
                    if constexpr (SHIFTED) b[r] = ld_src<SHIFTED>(s + 1);
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                if (r0 + r < N) {
                    float x[8];
                    unpack8(SHIFTED ? shift_bf16x8(a[r], b[r], D) : a[r], x);
                    if (r0 + r == 0) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] = x[e];
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], x[e]);
                    }
                }
            }
        }
    }
}

// The threads that share one unit: the whole CTA, or one warp (a unit of a
// pack); t is this thread's index among them.
struct Team {
    int t, n;
};

__device__ __forceinline__ Team cta_team() { return Team{(int)threadIdx.x, (int)blockDim.x}; }

template <int NR, bool SHIFTED, bool FP8, class Src>
__device__ __forceinline__ void fused_body(const Src& src_al, int N, int D, const FusedOut& o,
                                           int64_t k0, int nvec, bool avg, float fN,
                                           const AdamScalars& sc, float scale, float& mx,
                                           Team tm) {
#pragma unroll 1
    for (int q = tm.t; q < nvec; q += tm.n) {
        const int64_t k = k0 + 8 * (int64_t)q;
        float4 P[2], M[2], V[2];
        load_pmv8(o, k, P, M, V);
        float g[8];
        fold8<NR, SHIFTED>(src_al, N, q, D, g);
        if (avg) {
#pragma unroll
            for (int e = 0; e < 8; ++e) g[e] = div_n<NR>(g[e], fN);
        }
        fused8<FP8>(o, k, g, P, M, V, false, sc, scale, mx);
    }
}

// One real unit: fold, AdamW and the outputs of every element, peeled to an
// index that is a multiple of 8 (head / nvec vectors / tail).
template <int NR, bool FP8, class Src>
__device__ __forceinline__ void rs_adamw_real_unit(const Src& src_run, int N, const FusedOut& o,
                                                   int64_t k0, int len, int head, int nvec,
                                                   bool avg, float fN, const AdamScalars& sc,
                                                   float scale, float& mx,
                                                   Team tm = cta_team()) {
    const int done = head + 8 * nvec;
    if (tm.t < head)
        fused1<FP8>(o, k0 + tm.t, finish<NR>(fold_scalar<NR>(src_run.at(tm.t), N), avg, fN), false,
                    sc, scale, mx);
    // every rank's arena starts on a 16-byte boundary (P_arena % 8 == 0, and
    // table pointers are checked on the host), so one phase D holds for all N
    // source streams
    const int D = bf16_phase(src_run.rank(0) + head);
    const Src src_al = src_run.at(head - D);
    if (D == 0)
        fused_body<NR, false, FP8>(src_al, N, 0, o, k0 + head, nvec, avg, fN, sc, scale, mx, tm);
    else
        fused_body<NR, true, FP8>(src_al, N, D, o, k0 + head, nvec, avg, fN, sc, scale, mx, tm);
    if (tm.t < len - done)
        fused1<FP8>(o, k0 + done + tm.t,
                    finish<NR>(fold_scalar<NR>(src_run.at(done + tm.t), N), avg, fN), false, sc,
                    scale, mx);
}

// A pack of short real units and pad units, a warp per unit: the fused
// update of a group of thousands of small parameters, launched before
// k_rs_adamw, which then takes the long units only.  Same per-element
// arithmetic, so the same bits.  FP8: each warp folds its unit's max into the
// parameter's amax slot with one atomicMax.
template <int NR, bool FP8>
__global__ void __launch_bounds__(kThreads, 2)
k_rs_adamw_packs(const uint16_t* __restrict__ grads, int64_t stride, int N, FusedOut o,
                 const Unit* __restrict__ units, const int32_t* __restrict__ rpacks,
                 int64_t n_rpacks, int op_avg, AdamScalars sc,
                 const AdamScalars* __restrict__ sc_dev FSDPK_DBG_PARAM) {
    if ((int64_t)blockIdx.x >= n_rpacks) return;
    if (sc_dev != nullptr) sc = *sc_dev;  // scalars of a graph-replayed step
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    const int lane = threadIdx.x & 31;
    const Team tm{lane, 32};
    const int b = rpacks[blockIdx.x], e = rpacks[blockIdx.x + 1];
    for (int ui = b + (int)(threadIdx.x >> 5); ui < e; ui += kThreads / 32) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard | kChkArena);
        if constexpr (FP8)
            FSDPK_GUARD(u.is_pad || (o.unit_param[ui] >= 0 && o.unit_param[ui] < dbg.n_aux), ui);
        const int len = u.len;
        const int64_t k0 = u.shard_pos;
        float scale = 0.0f, mx = 0.0f;
        if constexpr (FP8) {
            if (!u.is_pad) scale = o.scales[o.unit_param[ui]];
        }
        int head = (int)((8 - (k0 & 7)) & 7);
        if (head > len) head = len;
        const int nvec = (len - head) >> 3;
        if (u.is_pad) {
            const int done = head + 8 * nvec;
            const float zero8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (lane < head) fused1<FP8>(o, k0 + lane, 0.0f, true, sc, scale, mx);
#pragma unroll 1
            for (int q = lane; q < nvec; q += 32) {
                const int64_t k = k0 + head + 8 * (int64_t)q;
                float4 P[2], M[2], V[2];
                load_pmv8(o, k, P, M, V);
                fused8<FP8>(o, k, zero8, P, M, V, true, sc, scale, mx);
            }
            if (lane < len - done) fused1<FP8>(o, k0 + done + lane, 0.0f, true, sc, scale, mx);
            continue;
        }
        rs_adamw_real_unit<NR, FP8>(StrideSrc{grads + u.arena_pos, stride}, N, o, k0, len, head,
                                    nvec, avg, fN, sc, scale, mx, tm);
        if constexpr (FP8) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            if (lane == 0) atomicMax(o.amax_bits + o.unit_param[ui], __float_as_uint(mx));
        }
    }
}

// TAB: the N source arenas come from a table of per-rank pointers (rank_tab,
// N <= kPeerMaxRanks) instead of grads + r * stride.  For 1 to 8 ranks, three
// CTAs per SM: the 80-register cap spills a few words at NR >= 6, and the
// fused kernel is still 0.7 % faster on B200 than with two CTAs and no spill.
// The any-N path would spill about 1 KB under that cap and keeps two.
template <int NR, bool FP8, bool TAB>
__global__ void __launch_bounds__(kThreads, (NR >= 1 && NR <= 8) ? 3 : 2)
k_rs_adamw(const uint16_t* __restrict__ grads, int64_t stride,
           const uint16_t* const* __restrict__ rank_tab, int N, FusedOut o,
           const Unit* __restrict__ units, int64_t n_units, int op_avg, AdamScalars sc,
           const AdamScalars* __restrict__ sc_dev FSDPK_DBG_PARAM) {
    __shared__ float part[kThreads / 32];
    __shared__ const uint16_t* s_tab[TAB ? kPeerMaxRanks : 1];
    if constexpr (TAB) load_rank_table(rank_tab, s_tab, N);
    if (sc_dev != nullptr) sc = *sc_dev;  // scalars of a graph-replayed step
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard | kChkArena);
        if constexpr (FP8)
            FSDPK_GUARD(u.is_pad || (o.unit_param[ui] >= 0 && o.unit_param[ui] < dbg.n_aux), ui);
        const int len = u.len;
        const int64_t k0 = u.shard_pos;
        float scale = 0.0f, mx = 0.0f;
        if constexpr (FP8) {
            if (!u.is_pad) scale = o.scales[o.unit_param[ui]];
        }
        // peel to an index that is a multiple of 8 (bf16 16-byte vectors)
        int head = (int)((8 - (k0 & 7)) & 7);
        if (head > len) head = len;
        const int nvec = (len - head) >> 3;
        if (u.is_pad) {
            const int done = head + 8 * nvec;
            const float zero8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if ((int)threadIdx.x < head) fused1<FP8>(o, k0 + threadIdx.x, 0.0f, true, sc, scale, mx);
#pragma unroll 1
            for (int q = threadIdx.x; q < nvec; q += blockDim.x) {
                const int64_t k = k0 + head + 8 * (int64_t)q;
                float4 P[2], M[2], V[2];
                load_pmv8(o, k, P, M, V);
                fused8<FP8>(o, k, zero8, P, M, V, true, sc, scale, mx);
            }
            if ((int)threadIdx.x < len - done)
                fused1<FP8>(o, k0 + done + threadIdx.x, 0.0f, true, sc, scale, mx);
            continue;
        }
        if constexpr (TAB)
            rs_adamw_real_unit<NR, FP8>(TableSrc{s_tab, u.arena_pos}, N, o, k0, len, head, nvec,
                                        avg, fN, sc, scale, mx);
        else
            rs_adamw_real_unit<NR, FP8>(StrideSrc{grads + u.arena_pos, stride}, N, o, k0, len,
                                        head, nvec, avg, fN, sc, scale, mx);
        if constexpr (FP8) {
            // the unit's max |updated master| into its parameter's amax slot
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = mx;
            __syncthreads();
            if (threadIdx.x < 32) {
                mx = threadIdx.x < kThreads / 32 ? part[threadIdx.x] : 0.0f;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                if (threadIdx.x == 0) atomicMax(o.amax_bits + o.unit_param[ui], __float_as_uint(mx));
            }
            __syncthreads();
        }
    }
}

// Flat fused update (a group of many small parameters, bf16 all-gather
// input): one CTA per tile of kFlatTile elements of [N][S], kFlatV vectors of
// 8 per thread with their codes read first.  A vector inside one real run
// loads master/m/v and every rank's 8 source elements at once, a pad vector
// updates with g = +0 and writes +0 to ag.  Mixed vectors go a thread per
// element.  Same per-element arithmetic as k_rs_adamw, so the same bits.
// This thread's elements of the mixed vectors (element t + i * T, T the
// region's threads, is element t % 8 of list entry t / 8), every load of all
// of them issued before the arithmetic.
template <int NR>
__device__ __forceinline__ void rs_adamw_flat_mixed(const uint16_t* __restrict__ grads,
                                                    int64_t stride, int N, const FusedOut& o,
                                                    int64_t count,
                                                    const int32_t* __restrict__ mixq,
                                                    const int32_t* __restrict__ mixc,
                                                    int64_t n_mixed, int64_t t0, int64_t T,
                                                    bool avg, float fN, const AdamScalars& sc
                                                    FSDPK_DBG_PARAM) {
    int64_t k[kFlatMixedPer];
    int32_t c[kFlatMixedPer];
    bool on[kFlatMixedPer];
    float pp[kFlatMixedPer], mm[kFlatMixedPer], vv[kFlatMixedPer];
#pragma unroll
    for (int i = 0; i < kFlatMixedPer; ++i) {
        const int64_t t = t0 + i * T;
        on[i] = t < 8 * n_mixed;
        k[i] = on[i] ? 8 * (int64_t)mixq[t >> 3] + (t & 7) : 0;
        c[i] = on[i] ? mixc[t] : kFlatPad;
        on[i] = on[i] && k[i] < count;
#ifdef FSDPK_DEBUG
        if (on[i] && !debug_ok_thread(dbg, k[i] < dbg.ns &&
                                               (c[i] == kFlatPad || (k[i] + (c[i] >> 1) >= 0 &&
                                                                     k[i] + (c[i] >> 1) < dbg.arena)),
                                      k[i]))
            on[i] = false;
#endif
        if (on[i]) {
            pp[i] = o.p[k[i]];
            mm[i] = o.m[k[i]];
            vv[i] = o.v[k[i]];
        }
    }
    float g[kFlatMixedPer];
    const int n = NR ? NR : N;
#pragma unroll
    for (int i = 0; i < kFlatMixedPer; ++i) g[i] = 0.0f;
#pragma unroll(NR ? NR : 1)
    for (int r = 0; r < n; ++r) {
        uint32_t h[kFlatMixedPer];
#pragma unroll
        for (int i = 0; i < kFlatMixedPer; ++i)
            h[i] = (on[i] && c[i] != kFlatPad) ? (uint32_t)grads[r * stride + k[i] + (c[i] >> 1)]
                                               : 0u;
#pragma unroll
        for (int i = 0; i < kFlatMixedPer; ++i)
            g[i] = r == 0 ? bf16_bits_to_f32(h[i]) : __fadd_rn(g[i], bf16_bits_to_f32(h[i]));
    }
#pragma unroll
    for (int i = 0; i < kFlatMixedPer; ++i) {
        if (!on[i]) continue;
        const bool pad = c[i] == kFlatPad;
        const float gi = pad ? 0.0f : finish<NR>(g[i], avg, fN);
        adamw1(pp[i], mm[i], vv[i], gi, sc);
        o.p[k[i]] = pp[i];
        o.m[k[i]] = mm[i];
        o.v[k[i]] = vv[i];
        if (o.red) o.red[k[i]] = gi;
        if (o.ag) {
            __nv_bfloat16 h = __float2bfloat16_rn(pad ? 0.0f : pp[i]);
            o.ag[k[i]] = *reinterpret_cast<uint16_t*>(&h);
        }
    }
}

// One launch: CTAs [0, mixed_ctas) take the mixed vectors' elements,
// kFlatMixedPer a thread, first in the grid; the others one tile each.
template <int NR>
__global__ void __launch_bounds__(kThreads, 2)
k_rs_adamw_flat(const uint16_t* __restrict__ grads, int64_t stride, int N, FusedOut o,
                int64_t count, const int32_t* __restrict__ smap, const int32_t* __restrict__ mixq,
                const int32_t* __restrict__ mixc, int64_t n_mixed, int64_t mixed_ctas,
                int op_avg, AdamScalars sc, const AdamScalars* __restrict__ sc_dev
                FSDPK_DBG_PARAM) {
    if (sc_dev != nullptr) sc = *sc_dev;  // scalars of a graph-replayed step
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    if ((int64_t)blockIdx.x < mixed_ctas) {
        rs_adamw_flat_mixed<NR>(grads, stride, N, o, count, mixq, mixc, n_mixed,
                                (int64_t)blockIdx.x * kThreads + threadIdx.x,
                                mixed_ctas * kThreads, avg, fN, sc FSDPK_DBG_ARG(dbg));
        return;
    }
    const int64_t nv = (count + 7) >> 3;
    const int64_t q0 = ((int64_t)blockIdx.x - mixed_ctas) * (kThreads * kFlatV) + threadIdx.x;
    int32_t code[kFlatV];
    flat_tile_codes(smap, q0, nv, code);
#pragma unroll 1
    for (int j = 0; j < kFlatV; ++j) {
        const int32_t c = flat_pick(code, j);
        if (c & 1) continue;  // mixed, or past the end
        const int64_t k = 8 * (q0 + (int64_t)j * kThreads);
        FSDPK_THREAD_GUARD(k + 8 <= count && k + 8 <= dbg.ns, k);
        float4 P[2], M[2], V[2];
        load_pmv8(o, k, P, M, V);
        float g[8];
        const bool pad = c == kFlatPad;
        if (pad) {
#pragma unroll
            for (int e = 0; e < 8; ++e) g[e] = 0.0f;
        } else {
            const int64_t a = k + (c >> 1);
            FSDPK_THREAD_GUARD(a >= 0 && a + 8 <= dbg.arena, k);
            flat_fold8<NR>(grads, stride, N, a, g);
            if (avg) {
#pragma unroll
                for (int e = 0; e < 8; ++e) g[e] = div_n<NR>(g[e], fN);
            }
        }
        float mx = 0.0f;
        fused8<false>(o, k, g, P, M, V, pad, sc, 0.0f, mx);
    }
}

// The fused update packs its short and pad units when there are at least
// this many of them (thousands of small parameters).
constexpr int64_t kFusedPackMinUnits = 2048;

template <int NR, bool FP8>
cudaError_t launch_rs_adamw_nr(const fsdp_group& g, const uint16_t* grads, const FusedOut& o,
                               int avg, const AdamScalars& sc, const AdamScalars* sc_dev,
                               cudaStream_t st) {
    if constexpr (!FP8) {
        if (g.flat) {
            const int64_t count = (int64_t)g.L * g.S;
            const int64_t n_mixed = (int64_t)g.smixq.size();
            const int64_t mixed_ctas = flat_mixed_ctas(n_mixed);
            k_rs_adamw_flat<NR><<<(unsigned)(flat_grid(count) + mixed_ctas), kThreads, 0, st>>>(
                grads, g.P_arena, g.N, o, count, g.d_smap, g.d_smixq, g.d_smixc, n_mixed,
                mixed_ctas, avg, sc, sc_dev FSDPK_DBG_ARG(debug_bounds(g, kDbgRsAdamwFlat)));
            return cudaGetLastError();
        }
    }
    int64_t nu = (int64_t)g.units.size();
    const int64_t n_small = nu - g.n_long_units;
    if (n_small >= kFusedPackMinUnits) {
        // thousands of short and pad units: packs first, then the long units
        const int64_t np = (int64_t)g.rpacks.size() - 1;
        k_rs_adamw_packs<NR, FP8><<<grid_for(g, nullptr, np), kThreads, 0, st>>>(
            grads, g.P_arena, g.N, o, g.d_units, g.d_rpacks, np, avg, sc, sc_dev
            FSDPK_DBG_ARG(debug_bounds(g, kDbgRsAdamw, g.n)));
        nu = g.n_long_units;
        if (nu == 0) return cudaGetLastError();
    }
    k_rs_adamw<NR, FP8, false><<<grid_for(g, nullptr, nu), kThreads, 0, st>>>(
        grads, g.P_arena, nullptr, g.N, o, g.d_units, nu, avg, sc, sc_dev
        FSDPK_DBG_ARG(debug_bounds(g, kDbgRsAdamw, g.n)));
    return cudaGetLastError();
}

template <bool FP8>
cudaError_t launch_rs_adamw_any(const fsdp_group& g, const uint16_t* grads, const FusedOut& o,
                                int avg, const AdamScalars& sc, const AdamScalars* sc_dev,
                                cudaStream_t st) {
    switch (g.N) {
#define FSDPK_CASE(K) \
    case K: return launch_rs_adamw_nr<K, FP8>(g, grads, o, avg, sc, sc_dev, st);
        FSDPK_CASE(1) FSDPK_CASE(2) FSDPK_CASE(3) FSDPK_CASE(4)
        FSDPK_CASE(5) FSDPK_CASE(6) FSDPK_CASE(7) FSDPK_CASE(8)
#undef FSDPK_CASE
        default:
            return launch_rs_adamw_nr<0, FP8>(g, grads, o, avg, sc, sc_dev, st);
    }
}

// One thread: advance the device step counter and compute that step's AdamW
// scalars in binary64, in the same operation order as the host path.
__global__ void k_adamw_prepare(double lr, double beta1, double beta2, double eps, double wd,
                                int64_t* __restrict__ step, AdamScalars* __restrict__ out) {
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    const int64_t t = *step + 1;
    *step = t;
    *out = adam_scalars_dev(lr, beta1, beta2, eps, wd, t);
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

cudaError_t launch_adamw(const fsdp_group& g, float* master, float* m, float* v,
                         const float* grad, const AdamScalars& sc, cudaStream_t st,
                         const AdamScalars* sc_dev) {
    const int64_t count = (int64_t)g.L * g.S;
    if (count == 0) return cudaSuccess;
    const int64_t items = ((count >> 2) + kAdamChunk4 - 1) / kAdamChunk4;
    k_adamw<<<grid_for(g, (const void*)k_adamw, items), kThreads, 0, st>>>(master, m, v, grad,
                                                                            count, sc, sc_dev);
    return cudaGetLastError();
}

cudaError_t launch_adamw_prepare(double lr, double beta1, double beta2, double eps, double wd,
                                 int64_t* step, AdamScalars* out, cudaStream_t st) {
    k_adamw_prepare<<<1, 32, 0, st>>>(lr, beta1, beta2, eps, wd, step, out);
    return cudaGetLastError();
}

cudaError_t launch_rs_adamw(const fsdp_group& g, const uint16_t* grads, int op, float* master,
                            float* m, float* v, const AdamScalars& sc, uint16_t* ag_next,
                            float* reduced, cudaStream_t st, const AdamScalars* sc_dev) {
    if (g.units.empty()) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    const FusedOut o{master, m, v, reduced, ag_next, nullptr, nullptr, nullptr, nullptr};
    return launch_rs_adamw_any<false>(g, grads, o, avg, sc, sc_dev, st);
}

cudaError_t launch_rs_adamw_fp8(const fsdp_group& g, const uint16_t* grads, int op, float* master,
                                float* m, float* v, const AdamScalars& sc, const float* scales_prev,
                                uint8_t* ag8_next, unsigned* amax_bits, float* reduced,
                                cudaStream_t st, const AdamScalars* sc_dev) {
    if (g.units.empty()) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    const FusedOut o{master, m, v, reduced, nullptr, ag8_next, scales_prev, amax_bits,
                     g.d_unit_param};
    return launch_rs_adamw_any<true>(g, grads, o, avg, sc, sc_dev, st);
}

template <int NR, bool FP8>
cudaError_t launch_rs_adamw_tab_nr(const fsdp_group& g, const uint16_t* const* tab,
                                   const FusedOut& o, int avg, const AdamScalars& sc,
                                   cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    k_rs_adamw<NR, FP8, true><<<grid_for(g, nullptr, nu), kThreads, 0, st>>>(
        nullptr, 0, tab, g.N, o, g.d_units, nu, avg, sc, nullptr
        FSDPK_DBG_ARG(debug_bounds(g, kDbgRsAdamwTab, g.n)));
    return cudaGetLastError();
}

template <bool FP8>
cudaError_t launch_rs_adamw_tab_any(const fsdp_group& g, const uint16_t* const* grad_tab,
                                    const FusedOut& o, int avg, const AdamScalars& sc,
                                    cudaStream_t st) {
    switch (g.N) {
#define FSDPK_CASE(K) \
    case K: return launch_rs_adamw_tab_nr<K, FP8>(g, grad_tab, o, avg, sc, st);
        FSDPK_CASE(1) FSDPK_CASE(2) FSDPK_CASE(3) FSDPK_CASE(4)
        FSDPK_CASE(5) FSDPK_CASE(6) FSDPK_CASE(7) FSDPK_CASE(8)
#undef FSDPK_CASE
        default:
            return launch_rs_adamw_tab_nr<0, FP8>(g, grad_tab, o, avg, sc, st);
    }
}

cudaError_t launch_rs_adamw_tab(const fsdp_group& g, const uint16_t* const* grad_tab, int op,
                                float* master, float* m, float* v, const AdamScalars& sc,
                                uint16_t* ag_next, float* reduced, cudaStream_t st) {
    if (g.units.empty()) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    const FusedOut o{master, m, v, reduced, ag_next, nullptr, nullptr, nullptr, nullptr};
    return launch_rs_adamw_tab_any<false>(g, grad_tab, o, avg, sc, st);
}

cudaError_t launch_rs_adamw_tab_fp8(const fsdp_group& g, const uint16_t* const* grad_tab, int op,
                                    float* master, float* m, float* v, const AdamScalars& sc,
                                    const float* scales_prev, uint8_t* ag8_next,
                                    unsigned* amax_bits, float* reduced, cudaStream_t st) {
    if (g.units.empty()) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    const FusedOut o{master, m, v, reduced, nullptr, ag8_next, scales_prev, amax_bits,
                     g.d_unit_param};
    return launch_rs_adamw_tab_any<true>(g, grad_tab, o, avg, sc, st);
}

}  // namespace fsdpk
