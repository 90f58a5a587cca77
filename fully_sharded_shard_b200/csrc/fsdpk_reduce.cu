// fsdpk_reduce.cu -- the reduce-scatter: per-rank bf16 gradients cast to
// reduce_dtype fp32, packed per destination rank and folded in rank order (SUM,
// AVG, or SUM then FSDP's own division), fused or through a materialised
// packed buffer; and gradient accumulation without sync with the
// reduce-scatter of the accumulated gradients.
//   "Introduction to PyTorch FSDP2 Backend Features", Mixed Precision;
//   "Sharded Training: FSDP2, DTensor, Tensor and Pipeline Parallelism",
//   Mixed precision and Other controls paragraphs, The bug Adam hid.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "fsdpk_device.cuh"

namespace fsdpk {
namespace {

// ---------------------------------------------------------------------------
// reduce-scatter, fused pack + rank-ordered reduction
// red[shard_pos + e] = ((g_0 + g_1) + ...) + g_{N-1}, g_r = fp32(grads[r][arena_pos + e])
// NR = ranks known at compile time (1..8), 0 = any N (batches of 4).
// ---------------------------------------------------------------------------

// The threads that share one unit: the whole CTA (a long unit) or one warp
// (a short or pad unit of a pack); t is this thread's index among them.
struct Team {
    int t, n;
};

__device__ __forceinline__ Team cta_team() { return Team{(int)threadIdx.x, (int)blockDim.x}; }

// Compile-time rank count: all NR loads of a vector are issued before the fold.
template <int NR, bool SHIFTED, int V, class Src>
__device__ __forceinline__ void reduce_body(const Src& src_al, float* __restrict__ dst, int nvec,
                                            int D, bool avg, float fN, Team tm) {
#pragma unroll 1
    for (int q0 = tm.t; q0 < nvec; q0 += tm.n * V) {
        uint4 a[V][NR];
        uint4 b[V][NR];
#pragma unroll
        for (int k = 0; k < V; ++k) {
            const int q = q0 + k * tm.n;
            if (q < nvec) {
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const uint4* s = reinterpret_cast<const uint4*>(src_al.rank(r)) + q;
                    a[k][r] = ld_src<SHIFTED>(s);
                    if constexpr (SHIFTED) b[k][r] = ld_src<SHIFTED>(s + 1);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < V; ++k) {
            const int q = q0 + k * tm.n;
            if (q < nvec) {
                float acc[8];
                unpack8(SHIFTED ? shift_bf16x8(a[k][0], b[k][0], D) : a[k][0], acc);
#pragma unroll
                for (int r = 1; r < NR; ++r) {
                    float x[8];
                    unpack8(SHIFTED ? shift_bf16x8(a[k][r], b[k][r], D) : a[k][r], x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], x[e]);
                }
                if (avg) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] = div_n<NR>(acc[e], fN);
                }
                store8(dst + 8 * q, acc);
            }
        }
    }
}

// Any rank count: ranks in batches of 4, folded in rank order.
template <bool SHIFTED, class Src>
__device__ __forceinline__ void reduce_body_any(const Src& src_al, int N,
                                                float* __restrict__ dst, int nvec, int D,
                                                bool avg, float fN, Team tm) {
#pragma unroll 1
    for (int q = tm.t; q < nvec; q += tm.n) {
        float acc[8];
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
        if (avg) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = __fdiv_rn(acc[e], fN);
        }
        store8(dst + 8 * q, acc);
    }
}

template <int NR, bool SHIFTED, class Src>
__device__ __forceinline__ void reduce_body_dispatch(const Src& src_al, int N, float* dst,
                                                     int nvec, int D, bool avg, float fN,
                                                     Team tm) {
    if constexpr (NR == 0) {
        reduce_body_any<SHIFTED>(src_al, N, dst, nvec, D, avg, fN, tm);
    } else {
        // keep about 4-8 independent 16-byte loads in flight per thread
        constexpr int V = NR >= 4 ? 1 : (4 / NR);
        reduce_body<NR, SHIFTED, V>(src_al, dst, nvec, D, avg, fN, tm);
    }
}

// One real unit: dst_run[e] = fold over ranks of src_run.rank(r)[e].
template <int NR, class Src>
__device__ __forceinline__ void reduce_unit(const Src& src_run, float* __restrict__ dst_run,
                                            int len, int N, bool avg, float fN,
                                            Team tm = cta_team()) {
    const int head = (int)head_to_16B(dst_run, len);
    if (tm.t < head)
        dst_run[tm.t] = finish<NR>(fold_scalar<NR>(src_run.at(tm.t), N), avg, fN);
    const int nvec = (len - head) >> 3;
    // every rank's arena starts on a 16-byte boundary (P_arena % 8 == 0, and
    // table pointers are checked on the host), so one phase D holds for all N
    // source streams
    const int D = bf16_phase(src_run.rank(0) + head);
    const Src src_al = src_run.at(head - D);
    float* dst = dst_run + head;
    if (D == 0) reduce_body_dispatch<NR, false>(src_al, N, dst, nvec, 0, avg, fN, tm);
    else reduce_body_dispatch<NR, true>(src_al, N, dst, nvec, D, avg, fN, tm);
    const int done = head + 8 * nvec;
    if (tm.t < len - done)
        dst_run[done + tm.t] = finish<NR>(fold_scalar<NR>(src_run.at(done + tm.t), N), avg, fN);
}

// Zero-fill `len` fp32 elements at dst (any alignment) by one warp.
__device__ __forceinline__ void zero_f32_warp(float* __restrict__ dst, int64_t len, int lane) {
    int64_t head = (4 - (reinterpret_cast<uintptr_t>(dst) >> 2 & 3)) & 3;
    if (head > len) head = len;
    if (lane < head) dst[lane] = 0.0f;
    const int64_t nv = (len - head) >> 2;
    float4* d4 = reinterpret_cast<float4*>(dst + head);
    for (int64_t q = lane; q < nv; q += 32) __stcs(d4 + q, make_float4(0.f, 0.f, 0.f, 0.f));
    const int64_t done = head + 4 * nv;
    if (lane < len - done) dst[done + lane] = 0.0f;
}

// A pack of short real units and pad units, a warp per unit: not inlined into
// k_reduce_units, so that its registers do not add to the long-unit path's.
template <int NR>
__device__ __noinline__ void reduce_pack(const uint16_t* __restrict__ gsrc, int64_t stride, int N,
                                         float* __restrict__ gdst, const Unit* __restrict__ units,
                                         int b, int e, bool avg, float fN FSDPK_DBG_PARAM) {
    const int lane = threadIdx.x & 31;
    for (int ui = b + (int)(threadIdx.x >> 5); ui < e; ui += kThreads / 32) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard | kChkArena);
        float* dst_run = gdst + u.shard_pos;
        if (u.is_pad) {
            zero_f32_warp(dst_run, u.len, lane);
            continue;
        }
        reduce_unit<NR>(StrideSrc{gsrc + u.arena_pos, stride}, dst_run, u.len, N, avg, fN,
                        Team{lane, 32});
    }
}

// One launch covers every unit of the group.  blockIdx.y selects a source
// rank for the pack kernel (NR == 1, src/dst offset per y); the fused
// reduction runs with gridDim.y == 1.  For 3 to 8 ranks, four CTAs per SM:
// the 64-register cap spills a few words at NR = 8, and the llama7b step is
// still 1.7 % faster on B200 than with three CTAs and no spill (more 16-byte
// loads in flight per SM).  The pack (NR = 1), NR = 2 and the any-N path
// would spill far more under that cap and keep three.
// PACKS: the grid starts with n_rpacks CTAs of packed short and pad units.
// Only a plan with many such units launches this form: the call to the pack
// path costs the long-unit path a few registers.
template <int NR, bool PACKS>
__global__ void __launch_bounds__(kThreads, (NR >= 3 && NR <= 8) ? 4 : 3)
k_reduce_units(const uint16_t* __restrict__ grads, int64_t stride, int N,
               float* __restrict__ out, int64_t y_src_step, int64_t y_dst_step,
               const Unit* __restrict__ units, int64_t n_units, int op_avg,
               const int32_t* __restrict__ rpacks, int64_t n_rpacks FSDPK_DBG_PARAM) {
    const uint16_t* gsrc = grads + (int64_t)blockIdx.y * y_src_step;
    float* gdst = out + (int64_t)blockIdx.y * y_dst_step;
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    // CTAs [0, n_rpacks): one pack of short or pad units each; the others one
    // unit of [0, n_units) each (the long units, or every unit without packs)
    if constexpr (PACKS) {
        if ((int64_t)blockIdx.x < n_rpacks) {
            const int p = (int)blockIdx.x;
            reduce_pack<NR>(gsrc, stride, N, gdst, units, rpacks[p], rpacks[p + 1], avg, fN
                            FSDPK_DBG_ARG(dbg));
            return;
        }
    } else {
        (void)rpacks;
    }
    for (int64_t ui = (int64_t)blockIdx.x - n_rpacks; ui < n_units;
         ui += (int64_t)gridDim.x - n_rpacks) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard | kChkArena);
        const int len = u.len;
        float* dst_run = gdst + u.shard_pos;
        if (u.is_pad) {
            zero_f32_run(dst_run, len);
            continue;
        }
        reduce_unit<NR>(StrideSrc{gsrc + u.arena_pos, stride}, dst_run, len, N, avg, fN);
    }
}

// The fused reduction with one source pointer per rank (a TableSrc):
// red[shard_pos + e] = fold_r fp32(rank_tab[r][arena_pos + e]).
template <int NR>
__global__ void __launch_bounds__(kThreads, (NR >= 3 && NR <= 8) ? 4 : 3)
k_reduce_units_tab(const uint16_t* const* __restrict__ rank_tab, int N, float* __restrict__ out,
                   const Unit* __restrict__ units, int64_t n_units, int op_avg FSDPK_DBG_PARAM) {
    __shared__ const uint16_t* s_tab[kPeerMaxRanks];
    load_rank_table(rank_tab, s_tab, N);
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard | kChkArena);
        float* dst_run = out + u.shard_pos;
        if (u.is_pad) {
            zero_f32_run(dst_run, u.len);
            continue;
        }
        reduce_unit<NR>(TableSrc{s_tab, u.arena_pos}, dst_run, u.len, N, avg, fN);
    }
}

// ---------------------------------------------------------------------------
// flat fused reduce-scatter (a group of many small parameters): one CTA per
// tile of kFlatTile elements of [N][S].  Each thread reads the codes of its
// kFlatV vectors first; a vector inside one real run folds its 8 elements
// from aligned 16-byte loads of every rank (shifted by the run's phase), a
// pad vector is +0.  Mixed vectors go a thread per element.  Same
// arithmetic per element as k_reduce_units, so the same bits.
// ---------------------------------------------------------------------------

// This thread's elements of the mixed vectors: element t + i * T (T the
// region's threads) is element e = t % 8 of list entry m = t / 8, i.e.
// k = 8 * mixq[m] + e with code mixc[t]; every rank's loads of all of them
// issued before the folds.
template <int NR>
__device__ __forceinline__ void reduce_flat_mixed(const uint16_t* __restrict__ grads,
                                                  int64_t stride, int N, float* __restrict__ out,
                                                  int64_t count, const int32_t* __restrict__ mixq,
                                                  const int32_t* __restrict__ mixc,
                                                  int64_t n_mixed, int64_t t0, int64_t T,
                                                  bool avg, float fN FSDPK_DBG_PARAM) {
    int64_t k[kFlatMixedPer];
    int32_t c[kFlatMixedPer];
    bool on[kFlatMixedPer];
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
    for (int i = 0; i < kFlatMixedPer; ++i)
        if (on[i]) out[k[i]] = c[i] == kFlatPad ? 0.0f : finish<NR>(g[i], avg, fN);
}

// One launch: CTAs [0, mixed_ctas) take the mixed vectors' elements,
// kFlatMixedPer a thread (first in the grid, so that these few latency-bound
// CTAs run beside the tiles rather than after them); the others one tile
// each.
template <int NR>
__global__ void __launch_bounds__(kThreads, (NR >= 1 && NR <= 8) ? 3 : 2)
k_reduce_flat(const uint16_t* __restrict__ grads, int64_t stride, int N, float* __restrict__ out,
              int64_t count, const int32_t* __restrict__ smap, const int32_t* __restrict__ mixq,
              const int32_t* __restrict__ mixc, int64_t n_mixed, int64_t mixed_ctas,
              int op_avg FSDPK_DBG_PARAM) {
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    if ((int64_t)blockIdx.x < mixed_ctas) {
        reduce_flat_mixed<NR>(grads, stride, N, out, count, mixq, mixc, n_mixed,
                              (int64_t)blockIdx.x * kThreads + threadIdx.x, mixed_ctas * kThreads,
                              avg, fN FSDPK_DBG_ARG(dbg));
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
        float acc[8];
        if (c == kFlatPad) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        } else {
            const int64_t a = k + (c >> 1);
            FSDPK_THREAD_GUARD(a >= 0 && a + 8 <= dbg.arena, k);
            flat_fold8<NR>(grads, stride, N, a, acc);
            if (avg) {
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = div_n<NR>(acc[e], fN);
            }
        }
        store8(out + k, acc);
    }
}

// ---------------------------------------------------------------------------
// staged reduce-scatter: reduce the materialised packed buffer
// red[k] = fold_r packed[r*NS + k]; then an optional separate division pass.
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kThreads)
k_reduce_packed_v4(const float* __restrict__ packed, int64_t NS, int N,
                   float* __restrict__ red, int64_t n4, int op_avg) {
    const float fN = (float)N;
    for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < n4;
         q += (int64_t)gridDim.x * blockDim.x) {
        float4 acc = __ldcs(reinterpret_cast<const float4*>(packed) + q);
        for (int r = 1; r < N; ++r) {
            float4 x = __ldcs(reinterpret_cast<const float4*>(packed + (int64_t)r * NS) + q);
            acc.x = __fadd_rn(acc.x, x.x);
            acc.y = __fadd_rn(acc.y, x.y);
            acc.z = __fadd_rn(acc.z, x.z);
            acc.w = __fadd_rn(acc.w, x.w);
        }
        if (op_avg) {
            acc.x = __fdiv_rn(acc.x, fN);
            acc.y = __fdiv_rn(acc.y, fN);
            acc.z = __fdiv_rn(acc.z, fN);
            acc.w = __fdiv_rn(acc.w, fN);
        }
        __stcs(reinterpret_cast<float4*>(red) + q, acc);
    }
}

// Scalar form for the elements not covered by 16-byte vectors (all of them
// when NS is not a multiple of 4, since rank streams are then misaligned).
__global__ void __launch_bounds__(kThreads)
k_reduce_packed_scalar(const float* __restrict__ packed, int64_t NS, int N,
                       float* __restrict__ red, int64_t begin, int op_avg) {
    const float fN = (float)N;
    for (int64_t k = begin + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < NS;
         k += (int64_t)gridDim.x * blockDim.x) {
        float acc = packed[k];
        for (int r = 1; r < N; ++r) acc = __fadd_rn(acc, packed[(int64_t)r * NS + k]);
        red[k] = op_avg ? __fdiv_rn(acc, fN) : acc;
    }
}

__global__ void __launch_bounds__(kThreads)
k_div_inplace(float* __restrict__ red, int64_t count, float fN) {
    for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < count;
         k += (int64_t)gridDim.x * blockDim.x)
        red[k] = __fdiv_rn(red[k], fN);
}

// ---------------------------------------------------------------------------
// gradient accumulation without sync, in reduce_dtype fp32
//   first: acc[k] = fp32(g[k]);  later: acc[k] = acc[k] + fp32(g[k])
// over the flat per-rank arenas [N][P_arena] (a multiple of 8 elements).
// ---------------------------------------------------------------------------

constexpr int kAccV = 2;  // 8-element vectors per thread per chunk
constexpr int64_t kAccChunk8 = (int64_t)kThreads * kAccV;

__global__ void __launch_bounds__(kThreads, 3)
k_accumulate(const uint16_t* __restrict__ g, float* __restrict__ acc, int64_t n8, int first) {
    const uint4* g8 = reinterpret_cast<const uint4*>(g);
    float4* a4 = reinterpret_cast<float4*>(acc);
    const int64_t n_chunks = (n8 + kAccChunk8 - 1) / kAccChunk8;
    for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x) {
        const int64_t q0 = c * kAccChunk8 + threadIdx.x;
        uint4 w[kAccV];
        float4 A[kAccV][2];
#pragma unroll
        for (int k = 0; k < kAccV; ++k) {
            const int64_t q = q0 + k * kThreads;
            if (q < n8) {
                w[k] = __ldcs(g8 + q);
                if (!first) {
                    A[k][0] = __ldcs(a4 + 2 * q);
                    A[k][1] = __ldcs(a4 + 2 * q + 1);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < kAccV; ++k) {
            const int64_t q = q0 + k * kThreads;
            if (q < n8) {
                float x[8];
                unpack8(w[k], x);
                if (!first) {
                    const float a[8] = {A[k][0].x, A[k][0].y, A[k][0].z, A[k][0].w,
                                        A[k][1].x, A[k][1].y, A[k][1].z, A[k][1].w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = __fadd_rn(a[e], x[e]);
                }
                __stcs(a4 + 2 * q, make_float4(x[0], x[1], x[2], x[3]));
                __stcs(a4 + 2 * q + 1, make_float4(x[4], x[5], x[6], x[7]));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// reduce-scatter of the accumulated gradients (the last microbatch)
//   red[shard_pos + e] = fold over r of x_r, x_r = acc_r[k] (+ fp32(g_r[k]))
// with k = arena_pos + e, the same rank-ordered fold and division as
// k_reduce_units.  A run whose source and destination are congruent mod 8
// moves 16-byte vectors; any other run goes element by element.
// ---------------------------------------------------------------------------

template <bool WITH_G>
__device__ __forceinline__ float acc_src1(const float* __restrict__ acc,
                                          const uint16_t* __restrict__ g, int64_t k) {
    float x = acc[k];
    if constexpr (WITH_G) x = __fadd_rn(x, bf16_bits_to_f32(g[k]));
    return x;
}

template <bool WITH_G>
__global__ void __launch_bounds__(kThreads, 2)
k_reduce_acc(const float* __restrict__ acc, const uint16_t* __restrict__ g, int64_t stride, int N,
             float* __restrict__ out, const Unit* __restrict__ units, int64_t n_units,
             int op_avg FSDPK_DBG_PARAM) {
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard | kChkArena);
        const int len = u.len;
        float* dst = out + u.shard_pos;
        if (u.is_pad) {
            zero_f32_run(dst, len);
            continue;
        }
        const int64_t s0 = u.arena_pos;
        const bool vec = ((s0 - u.shard_pos) & 7) == 0;
        int head = vec ? (int)((8 - (s0 & 7)) & 7) : len;
        if (head > len) head = len;
        for (int e = threadIdx.x; e < head; e += blockDim.x) {
            float a = acc_src1<WITH_G>(acc, g, s0 + e);
            for (int r = 1; r < N; ++r)
                a = __fadd_rn(a, acc_src1<WITH_G>(acc, g, (int64_t)r * stride + s0 + e));
            dst[e] = finish(a, avg, fN);
        }
        const int nvec = (len - head) >> 3;
#pragma unroll 1
        for (int q = threadIdx.x; q < nvec; q += blockDim.x) {
            const int64_t k = s0 + head + 8 * (int64_t)q;
            float accv[8];
#pragma unroll 1
            for (int r0 = 0; r0 < N; r0 += 4) {
                float4 A[4][2];
                uint4 w[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    if (r0 + r < N) {
                        const int64_t kr = (int64_t)(r0 + r) * stride + k;
                        A[r][0] = __ldcs(reinterpret_cast<const float4*>(acc + kr));
                        A[r][1] = __ldcs(reinterpret_cast<const float4*>(acc + kr) + 1);
                        if constexpr (WITH_G) w[r] = __ldcs(reinterpret_cast<const uint4*>(g + kr));
                    }
                }
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    if (r0 + r < N) {
                        float x[8] = {A[r][0].x, A[r][0].y, A[r][0].z, A[r][0].w,
                                      A[r][1].x, A[r][1].y, A[r][1].z, A[r][1].w};
                        if constexpr (WITH_G) {
                            float y[8];
                            unpack8(w[r], y);
#pragma unroll
                            for (int e = 0; e < 8; ++e) x[e] = __fadd_rn(x[e], y[e]);
                        }
                        if (r0 + r == 0) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) accv[e] = x[e];
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) accv[e] = __fadd_rn(accv[e], x[e]);
                        }
                    }
                }
            }
            if (avg) {
#pragma unroll
                for (int e = 0; e < 8; ++e) accv[e] = __fdiv_rn(accv[e], fN);
            }
            store8(dst + head + 8 * q, accv);
        }
        const int done = head + 8 * nvec;
        for (int e = done + threadIdx.x; e < len; e += blockDim.x) {
            float a = acc_src1<WITH_G>(acc, g, s0 + e);
            for (int r = 1; r < N; ++r)
                a = __fadd_rn(a, acc_src1<WITH_G>(acc, g, (int64_t)r * stride + s0 + e));
            dst[e] = finish(a, avg, fN);
        }
    }
}

// n_units: the units one CTA each handles; rpacks / n_rpacks: the packs
// (null / 0 when every unit gets a CTA).
template <int NR>
cudaError_t launch_reduce_nr(const fsdp_group& g, const uint16_t* grads, int64_t stride, int N,
                             float* out, int64_t y_src_step, int64_t y_dst_step,
                             unsigned ydim, const Unit* units, int64_t n_units, int avg,
                             cudaStream_t st, const DebugBounds& dbg,
                             const int32_t* rpacks = nullptr, int64_t n_rpacks = 0) {
    (void)dbg;
    dim3 grid(grid_for(g, nullptr, n_rpacks + n_units), ydim);
    if (n_rpacks > 0)
        k_reduce_units<NR, true><<<grid, kThreads, 0, st>>>(grads, stride, N, out, y_src_step,
                                                            y_dst_step, units, n_units, avg,
                                                            rpacks, n_rpacks FSDPK_DBG_ARG(dbg));
    else
        k_reduce_units<NR, false><<<grid, kThreads, 0, st>>>(grads, stride, N, out, y_src_step,
                                                             y_dst_step, units, n_units, avg,
                                                             nullptr, 0 FSDPK_DBG_ARG(dbg));
    return cudaGetLastError();
}

// The reduce-scatter packs its short and pad units when there are at least
// this many of them (thousands of small parameters); otherwise every unit
// gets a CTA of the plain kernel.
constexpr int64_t kPackMinUnits = 2048;

// (units a CTA each, packs) of g for the fused reduce-scatter kernels.
inline void reduce_split(const fsdp_group& g, int64_t* n_cta_units, int64_t* n_packs) {
    const int64_t n_small = (int64_t)g.units.size() - g.n_long_units;
    if (n_small >= kPackMinUnits) {
        *n_cta_units = g.n_long_units;
        *n_packs = (int64_t)g.rpacks.size() - 1;
    } else {
        *n_cta_units = (int64_t)g.units.size();
        *n_packs = 0;
    }
}

template <int NR>
cudaError_t launch_reduce_flat_nr(const fsdp_group& g, const uint16_t* grads, int avg,
                                  float* reduced, cudaStream_t st) {
    const int64_t count = (int64_t)g.L * g.S;
    const int64_t n_mixed = (int64_t)g.smixq.size();
    const int64_t mixed_ctas = flat_mixed_ctas(n_mixed);
    k_reduce_flat<NR><<<(unsigned)(flat_grid(count) + mixed_ctas), kThreads, 0, st>>>(
        grads, g.P_arena, g.N, reduced, count, g.d_smap, g.d_smixq, g.d_smixc, n_mixed,
        mixed_ctas, avg FSDPK_DBG_ARG(debug_bounds(g, kDbgReduceFlat)));
    return cudaGetLastError();
}

// The flat fused reduce-scatter of a plan with the flat tables.
cudaError_t launch_reduce_flat(const fsdp_group& g, const uint16_t* grads, int avg,
                               float* reduced, cudaStream_t st) {
    switch (g.N) {
#define FSDPK_CASE(K) \
    case K: return launch_reduce_flat_nr<K>(g, grads, avg, reduced, st);
        FSDPK_CASE(1) FSDPK_CASE(2) FSDPK_CASE(3) FSDPK_CASE(4)
        FSDPK_CASE(5) FSDPK_CASE(6) FSDPK_CASE(7) FSDPK_CASE(8)
#undef FSDPK_CASE
        default:
            return launch_reduce_flat_nr<0>(g, grads, avg, reduced, st);
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

cudaError_t launch_rs_fused(const fsdp_group& g, const uint16_t* grads, int op, float* reduced,
                            cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    if (nu == 0) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    const int64_t stride = g.P_arena;
    const DebugBounds dbg = debug_bounds(g, kDbgReduce);
    if (g.flat) return launch_reduce_flat(g, grads, avg, reduced, st);
    int64_t nl, np;
    reduce_split(g, &nl, &np);
    (void)nu;
    switch (g.N) {
#define FSDPK_CASE(K) \
    case K: return launch_reduce_nr<K>(g, grads, stride, g.N, reduced, 0, 0, 1, g.d_units, nl, avg, st, dbg, g.d_rpacks, np);
        FSDPK_CASE(1) FSDPK_CASE(2) FSDPK_CASE(3) FSDPK_CASE(4)
        FSDPK_CASE(5) FSDPK_CASE(6) FSDPK_CASE(7) FSDPK_CASE(8)
#undef FSDPK_CASE
        default:
            return launch_reduce_nr<0>(g, grads, stride, g.N, reduced, 0, 0, 1, g.d_units, nl, avg,
                                       st, dbg, g.d_rpacks, np);
    }
}

cudaError_t launch_rs_fused_units(int sm_count, int N, int64_t P_arena, const Unit* units,
                                  int64_t n_units, const uint16_t* grads, int op, float* reduced,
                                  cudaStream_t st, int64_t NS) {
    if (n_units == 0) return cudaSuccess;
    fsdp_group g;  // only the SM count is read when sizing the grid
    g.sm_count = sm_count;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    const DebugBounds dbg = debug_bounds_raw(NS, P_arena, kDbgReduce);
    switch (N) {
#define FSDPK_CASE(K) \
    case K: return launch_reduce_nr<K>(g, grads, P_arena, N, reduced, 0, 0, 1, units, n_units, avg, st, dbg);
        FSDPK_CASE(1) FSDPK_CASE(2) FSDPK_CASE(3) FSDPK_CASE(4)
        FSDPK_CASE(5) FSDPK_CASE(6) FSDPK_CASE(7) FSDPK_CASE(8)
#undef FSDPK_CASE
        default:
            return launch_reduce_nr<0>(g, grads, P_arena, N, reduced, 0, 0, 1, units, n_units, avg,
                                       st, dbg);
    }
}

template <int NR>
cudaError_t launch_reduce_tab_nr(const fsdp_group& g, const uint16_t* const* tab, float* out,
                                 int avg, cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    k_reduce_units_tab<NR><<<grid_for(g, nullptr, nu), kThreads, 0, st>>>(
        tab, g.N, out, g.d_units, nu, avg FSDPK_DBG_ARG(debug_bounds(g, kDbgReduceTab)));
    return cudaGetLastError();
}

cudaError_t launch_rs_fused_tab(const fsdp_group& g, const uint16_t* const* grad_tab, int op,
                                float* reduced, cudaStream_t st) {
    if (g.units.empty()) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    switch (g.N) {
#define FSDPK_CASE(K) \
    case K: return launch_reduce_tab_nr<K>(g, grad_tab, reduced, avg, st);
        FSDPK_CASE(1) FSDPK_CASE(2) FSDPK_CASE(3) FSDPK_CASE(4)
        FSDPK_CASE(5) FSDPK_CASE(6) FSDPK_CASE(7) FSDPK_CASE(8)
#undef FSDPK_CASE
        default:
            return launch_reduce_tab_nr<0>(g, grad_tab, reduced, avg, st);
    }
}

cudaError_t launch_rs_pack(const fsdp_group& g, const uint16_t* grads, float* packed,
                           cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    if (nu == 0) return cudaSuccess;
    // blockIdx.y = source rank r: reads rank r's arena, writes packed[r]
    int64_t nl, np;
    reduce_split(g, &nl, &np);
    return launch_reduce_nr<1>(g, grads, 0, 1, packed, g.P_arena, (int64_t)g.N * g.S,
                               (unsigned)g.N, g.d_units, nl, 0, st, debug_bounds(g, kDbgReduce),
                               g.d_rpacks, np);
}

cudaError_t launch_rs_reduce_packed(const fsdp_group& g, const float* packed, int op,
                                    float* reduced, cudaStream_t st) {
    const int64_t NS = (int64_t)g.N * g.S;
    if (NS == 0) return cudaSuccess;
    const int avg = (op == FSDP_AVG) ? 1 : 0;
    int64_t begin = 0;
    if (NS % 4 == 0) {
        const int64_t n4 = NS / 4;
        k_reduce_packed_v4<<<grid_for(g, (const void*)k_reduce_packed_v4, (n4 + kThreads - 1) / kThreads),
                             kThreads, 0, st>>>(packed, NS, g.N, reduced, n4, avg);
        begin = NS;
    }
    if (begin < NS) {
        k_reduce_packed_scalar<<<grid_for(g, (const void*)k_reduce_packed_scalar,
                                          (NS - begin + kThreads - 1) / kThreads),
                                 kThreads, 0, st>>>(packed, NS, g.N, reduced, begin, avg);
    }
    return cudaGetLastError();
}

cudaError_t launch_div_inplace(const fsdp_group& g, float* reduced, cudaStream_t st) {
    const int64_t NS = (int64_t)g.N * g.S;
    if (NS == 0) return cudaSuccess;
    k_div_inplace<<<grid_for(g, (const void*)k_div_inplace, (NS + kThreads - 1) / kThreads),
                    kThreads, 0, st>>>(reduced, NS, (float)g.N);
    return cudaGetLastError();
}

cudaError_t launch_accumulate(const fsdp_group& g, const uint16_t* grads, float* acc, int first,
                              cudaStream_t st) {
    const int64_t n8 = (int64_t)g.N * g.P_arena / 8;
    if (n8 == 0) return cudaSuccess;
    const int64_t chunks = (n8 + kAccChunk8 - 1) / kAccChunk8;
    k_accumulate<<<grid_for(g, (const void*)k_accumulate, chunks), kThreads, 0, st>>>(grads, acc,
                                                                                     n8, first);
    return cudaGetLastError();
}

cudaError_t launch_rs_reduce_acc(const fsdp_group& g, const uint16_t* grads, const float* acc,
                                 int op, float* reduced, cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    if (nu == 0) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    if (grads != nullptr)
        k_reduce_acc<true><<<grid_for(g, (const void*)k_reduce_acc<true>, nu), kThreads, 0, st>>>(
            acc, grads, g.P_arena, g.N, reduced, g.d_units, nu, avg
            FSDPK_DBG_ARG(debug_bounds(g, kDbgReduceAcc)));
    else
        k_reduce_acc<false><<<grid_for(g, (const void*)k_reduce_acc<false>, nu), kThreads, 0, st>>>(
            acc, grads, g.P_arena, g.N, reduced, g.d_units, nu, avg
            FSDPK_DBG_ARG(debug_bounds(g, kDbgReduceAcc)));
    return cudaGetLastError();
}

}  // namespace fsdpk
