// fsdpk_kernels.cu -- sm_100a kernels of the FSDP2 per-parameter sharding
// step.  Every stage is HBM-bound streaming (well under one flop per byte), so
// nothing here uses tensor cores: the design goals are 16-byte coalesced
// accesses, enough bytes in flight per SM to cover HBM latency, streaming
// (evict-first) cache hints for data touched once, and grids sized to the
// SM count.
//
// Stages, by page title and section:
//   copy-in   -- "Sharded Training: FSDP2, DTensor, Tensor and Pipeline
//                Parallelism", Mixed precision paragraph: bf16 copies of the
//                fp32 shards are all-gathered.
//   copy-out  -- "Introduction to PyTorch FSDP2 Backend Features", Working
//                Principle (All-Gather state): shards become full parameters.
//   rs pack + reduce -- same pages: gradients cast to fp32 (reduce_dtype) and
//                reduce-scattered; AVG, or SUM plus FSDP's own division
//                (Sharded Training page, Other controls paragraph).
//   AdamW     -- Sharded Training page, Fence 4: the optimizer steps the
//                sharded fp32 parameters, its state sharded the same way.
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

// ---------------------------------------------------------------------------
// copy-in: ag[k] = bf16_rn(master[k]) for real elements, +0 in pad rows
// ---------------------------------------------------------------------------

// Bit i set when element k0+i lies in a pad interval.  Intervals in
// [rb, re) are sorted and disjoint; at most 8 of them can meet [k0, k0+8).
__device__ __forceinline__ uint32_t pad_mask8(int64_t k0, const Interval* __restrict__ iv,
                                              int rb, int re) {
    // first interval with hi > k0
    int lo = rb, hi = re;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if (iv[mid].hi > k0) hi = mid; else lo = mid + 1;
    }
    uint32_t mask = 0;
    for (int t = lo; t < re; ++t) {
        int64_t a = iv[t].lo, b = iv[t].hi;
        if (a >= k0 + 8) break;
        int64_t s = a > k0 ? a - k0 : 0;
        int64_t e = b < k0 + 8 ? b - k0 : 8;
        mask |= ((1u << e) - 1u) & ~((1u << s) - 1u);
    }
    return mask;
}

constexpr int kCopyInV = 4;  // vectors of 8 per thread per tile
static_assert(kCopyInTile == kThreads * 8 * kCopyInV, "copy-in tile shape");

__global__ void __launch_bounds__(kThreads)
k_copy_in(const float* __restrict__ master, uint16_t* __restrict__ ag, int64_t count,
          int64_t n_tiles, const Interval* __restrict__ iv,
          const TileRange* __restrict__ tr) {
    for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x) {
        const int64_t base = t * kCopyInTile;
        const int64_t end = min(base + kCopyInTile, count);
        TileRange rng{0, 0};
        if (tr != nullptr) rng = tr[t];
        float4 x[kCopyInV][2];
#pragma unroll
        for (int j = 0; j < kCopyInV; ++j) {
            const int64_t k = base + 8 * (threadIdx.x + (int64_t)j * kThreads);
            if (k + 8 <= end) {
                const float4* src = reinterpret_cast<const float4*>(master + k);
                x[j][0] = __ldcs(src);
                x[j][1] = __ldcs(src + 1);
            }
        }
#pragma unroll
        for (int j = 0; j < kCopyInV; ++j) {
            const int64_t k = base + 8 * (threadIdx.x + (int64_t)j * kThreads);
            if (k + 8 <= end) {
                float f[8] = {x[j][0].x, x[j][0].y, x[j][0].z, x[j][0].w,
                              x[j][1].x, x[j][1].y, x[j][1].z, x[j][1].w};
                if (rng.begin < rng.end) {
                    uint32_t mk = pad_mask8(k, iv, rng.begin, rng.end);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (mk & (1u << e)) f[e] = 0.0f;
                }
                uint4 o = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                     pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
                __stcs(reinterpret_cast<uint4*>(ag + k), o);
            } else if (k < end) {
                // ragged tail of the whole buffer: element by element
                for (int64_t q = k; q < end; ++q) {
                    float f = master[q];
                    if (rng.begin < rng.end && (pad_mask8(q, iv, rng.begin, rng.end) & 1u))
                        f = 0.0f;
                    __nv_bfloat16 h = __float2bfloat16_rn(f);
                    ag[q] = *reinterpret_cast<uint16_t*>(&h);
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// segment units: shared unit loop
// ---------------------------------------------------------------------------

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

// ---------------------------------------------------------------------------
// copy-out: arena[arena_pos + e] = ag[shard_pos + e] for each real unit
// ---------------------------------------------------------------------------

template <bool SHIFTED>
__device__ __forceinline__ void copy_out_body(const uint16_t* __restrict__ src_al,
                                              uint16_t* __restrict__ dst, int nvec, int D) {
    constexpr int V = SHIFTED ? 2 : 4;
    const uint4* s = reinterpret_cast<const uint4*>(src_al);
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll 1
    for (int q0 = threadIdx.x; q0 < nvec; q0 += blockDim.x * V) {
        uint4 a[V], b[V];
#pragma unroll
        for (int k = 0; k < V; ++k) {
            const int q = q0 + k * blockDim.x;
            if (q < nvec) {
                a[k] = ld_src<SHIFTED>(s + q);
                if constexpr (SHIFTED) b[k] = ld_src<SHIFTED>(s + q + 1);
            }
        }
#pragma unroll
        for (int k = 0; k < V; ++k) {
            const int q = q0 + k * blockDim.x;
            if (q < nvec) {
                uint4 o;
                if constexpr (SHIFTED) o = shift_bf16x8(a[k], b[k], D);
                else o = a[k];
                __stcs(d + q, o);
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 5)
k_copy_out(const uint16_t* __restrict__ ag, uint16_t* __restrict__ arena,
           const Unit* __restrict__ units, int64_t n_units) {
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        const int len = u.len;
        uint16_t* dst_run = arena + u.arena_pos;
        const uint16_t* src_run = ag + u.shard_pos;
        const int head = (int)head_to_16B(dst_run, len);
        if ((int)threadIdx.x < head) dst_run[threadIdx.x] = src_run[threadIdx.x];
        const int nvec = (len - head) >> 3;
        const int D = bf16_phase(src_run + head);
        const uint16_t* src_al = src_run + head - D;
        uint16_t* dst = dst_run + head;
        if (D == 0) copy_out_body<false>(src_al, dst, nvec, 0);
        else copy_out_body<true>(src_al, dst, nvec, D);
        const int done = head + 8 * nvec;
        if ((int)threadIdx.x < len - done) dst_run[done + threadIdx.x] = src_run[done + threadIdx.x];
    }
}

// ---------------------------------------------------------------------------
// reduce-scatter, fused pack + rank-ordered reduction
// red[shard_pos + e] = ((g_0 + g_1) + ...) + g_{N-1}, g_r = fp32(grads[r][arena_pos + e])
// NR = ranks known at compile time (1..8), 0 = any N (batches of 4).
// ---------------------------------------------------------------------------

template <int NR>
__device__ __forceinline__ float fold_scalar(const uint16_t* __restrict__ src, int64_t stride,
                                             int N) {
    const int n = NR ? NR : N;
    float acc = bf16_bits_to_f32(src[0]);
    for (int r = 1; r < n; ++r) acc = __fadd_rn(acc, bf16_bits_to_f32(src[r * stride]));
    return acc;
}

__device__ __forceinline__ float finish(float acc, bool avg, float fN) {
    return avg ? __fdiv_rn(acc, fN) : acc;
}

__device__ __forceinline__ void store8(float* __restrict__ dst, const float (&acc)[8]) {
    float4* o = reinterpret_cast<float4*>(dst);
    __stcs(o, make_float4(acc[0], acc[1], acc[2], acc[3]));
    __stcs(o + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
}

// Compile-time rank count: all NR loads of a vector are issued before the fold.
template <int NR, bool SHIFTED, int V>
__device__ __forceinline__ void reduce_body(const uint16_t* __restrict__ src_al, int64_t stride,
                                            float* __restrict__ dst, int nvec, int D, bool avg,
                                            float fN) {
#pragma unroll 1
    for (int q0 = threadIdx.x; q0 < nvec; q0 += blockDim.x * V) {
        uint4 a[V][NR];
        uint4 b[V][NR];
#pragma unroll
        for (int k = 0; k < V; ++k) {
            const int q = q0 + k * blockDim.x;
            if (q < nvec) {
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const uint4* s = reinterpret_cast<const uint4*>(src_al + r * stride) + q;
                    a[k][r] = ld_src<SHIFTED>(s);
                    if constexpr (SHIFTED) b[k][r] = ld_src<SHIFTED>(s + 1);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < V; ++k) {
            const int q = q0 + k * blockDim.x;
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
                    for (int e = 0; e < 8; ++e) acc[e] = __fdiv_rn(acc[e], fN);
                }
                store8(dst + 8 * q, acc);
            }
        }
    }
}

// Any rank count: ranks in batches of 4, folded in rank order.
template <bool SHIFTED>
__device__ __forceinline__ void reduce_body_any(const uint16_t* __restrict__ src_al,
                                                int64_t stride, int N,
                                                float* __restrict__ dst, int nvec, int D,
                                                bool avg, float fN) {
#pragma unroll 1
    for (int q = threadIdx.x; q < nvec; q += blockDim.x) {
        float acc[8];
#pragma unroll 1
        for (int r0 = 0; r0 < N; r0 += 4) {
            uint4 a[4], b[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                if (r0 + r < N) {
                    const uint4* s =
                        reinterpret_cast<const uint4*>(src_al + (int64_t)(r0 + r) * stride) + q;
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

template <int NR, bool SHIFTED>
__device__ __forceinline__ void reduce_body_dispatch(const uint16_t* src_al, int64_t stride,
                                                     int N, float* dst, int nvec, int D, bool avg,
                                                     float fN) {
    if constexpr (NR == 0) {
        reduce_body_any<SHIFTED>(src_al, stride, N, dst, nvec, D, avg, fN);
    } else {
        // keep about 4-8 independent 16-byte loads in flight per thread
        constexpr int V = NR >= 4 ? 1 : (4 / NR);
        reduce_body<NR, SHIFTED, V>(src_al, stride, dst, nvec, D, avg, fN);
    }
}

// One launch covers every unit of the group.  blockIdx.y selects a source
// rank for the pack kernel (NR == 1, src/dst offset per y); the fused
// reduction runs with gridDim.y == 1.
template <int NR>
__global__ void __launch_bounds__(kThreads, 3)
k_reduce_units(const uint16_t* __restrict__ grads, int64_t stride, int N,
               float* __restrict__ out, int64_t y_src_step, int64_t y_dst_step,
               const Unit* __restrict__ units, int64_t n_units, int op_avg) {
    const uint16_t* gsrc = grads + (int64_t)blockIdx.y * y_src_step;
    float* gdst = out + (int64_t)blockIdx.y * y_dst_step;
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        const int len = u.len;
        float* dst_run = gdst + u.shard_pos;
        if (u.is_pad) {
            zero_f32_run(dst_run, len);
            continue;
        }
        const uint16_t* src_run = gsrc + u.arena_pos;
        const int head = (int)head_to_16B(dst_run, len);
        if ((int)threadIdx.x < head)
            dst_run[threadIdx.x] =
                finish(fold_scalar<NR>(src_run + threadIdx.x, stride, N), avg, fN);
        const int nvec = (len - head) >> 3;
        // every rank's arena starts on a 16-byte boundary (P_arena % 8 == 0),
        // so one phase D holds for all N source streams
        const int D = bf16_phase(src_run + head);
        const uint16_t* src_al = src_run + head - D;
        float* dst = dst_run + head;
        if (D == 0) reduce_body_dispatch<NR, false>(src_al, stride, N, dst, nvec, 0, avg, fN);
        else reduce_body_dispatch<NR, true>(src_al, stride, N, dst, nvec, D, avg, fN);
        const int done = head + 8 * nvec;
        if ((int)threadIdx.x < len - done)
            dst_run[done + threadIdx.x] =
                finish(fold_scalar<NR>(src_run + done + threadIdx.x, stride, N), avg, fN);
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
// AdamW over the flat [N][S] buffers (pads are zero and stay zero)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void adamw1(float& p, float& m, float& v, float g,
                                       const AdamScalars& sc) {
    p = p * sc.decay;
    m = fmaf(sc.beta1, m, sc.omb1 * g);
    v = fmaf(sc.beta2, v, sc.omb2 * g * g);
    const float denom = fmaf(__fsqrt_rn(v), sc.inv_bc2_sqrt, sc.eps);
    p = fmaf(-sc.step_size, __fdiv_rn(m, denom), p);
}

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
// shard: master[shard_pos + e] = full[arena_pos + e]; pads +0 (set-up path)
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kThreads)
k_shard(const float* __restrict__ full, float* __restrict__ master,
        const Unit* __restrict__ units, int64_t n_units) {
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        if (u.is_pad) {
            zero_f32_run(master + u.shard_pos, u.len);
            continue;
        }
        for (int64_t e = threadIdx.x; e < u.len; e += blockDim.x)
            master[u.shard_pos + e] = full[u.arena_pos + e];
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
// ---------------------------------------------------------------------------

struct FusedOut {
    float* p;
    float* m;
    float* v;
    float* red;    // may be null
    uint16_t* ag;  // may be null
};

// One element: adamw with g, then the optional outputs.
__device__ __forceinline__ void fused1(const FusedOut& o, int64_t k, float g, bool pad,
                                       const AdamScalars& sc) {
    float pp = o.p[k], mm = o.m[k], vv = o.v[k];
    adamw1(pp, mm, vv, g, sc);
    o.p[k] = pp;
    o.m[k] = mm;
    o.v[k] = vv;
    if (o.red) o.red[k] = g;
    if (o.ag) {
        __nv_bfloat16 h = __float2bfloat16_rn(pad ? 0.0f : pp);
        o.ag[k] = *reinterpret_cast<uint16_t*>(&h);
    }
}

// Eight elements starting at an index that is a multiple of 8 (every fp32
// pointer 32-byte aligned, the bf16 pointer 16-byte aligned).
__device__ __forceinline__ void fused8(const FusedOut& o, int64_t k, const float (&g)[8],
                                       const float4 (&P)[2], const float4 (&M)[2],
                                       const float4 (&V)[2], bool pad, const AdamScalars& sc) {
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
    if (o.ag) {
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
template <int NR, bool SHIFTED>
__device__ __forceinline__ void fold8(const uint16_t* __restrict__ src_al, int64_t stride, int N,
                                      int q, int D, float (&acc)[8]) {
    if constexpr (NR != 0) {
        uint4 a[NR], b[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            const uint4* s = reinterpret_cast<const uint4*>(src_al + r * stride) + q;
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
                    const uint4* s =
                        reinterpret_cast<const uint4*>(src_al + (int64_t)(r0 + r) * stride) + q;
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

template <int NR, bool SHIFTED>
__device__ __forceinline__ void fused_body(const uint16_t* __restrict__ src_al, int64_t stride,
                                           int N, int D, const FusedOut& o, int64_t k0, int nvec,
                                           bool avg, float fN, const AdamScalars& sc) {
#pragma unroll 1
    for (int q = threadIdx.x; q < nvec; q += blockDim.x) {
        const int64_t k = k0 + 8 * (int64_t)q;
        float4 P[2], M[2], V[2];
        load_pmv8(o, k, P, M, V);
        float g[8];
        fold8<NR, SHIFTED>(src_al, stride, N, q, D, g);
        if (avg) {
#pragma unroll
            for (int e = 0; e < 8; ++e) g[e] = __fdiv_rn(g[e], fN);
        }
        fused8(o, k, g, P, M, V, false, sc);
    }
}

template <int NR>
__global__ void __launch_bounds__(kThreads, 2)
k_rs_adamw(const uint16_t* __restrict__ grads, int64_t stride, int N, FusedOut o,
           const Unit* __restrict__ units, int64_t n_units, int op_avg, AdamScalars sc,
           const AdamScalars* __restrict__ sc_dev) {
    if (sc_dev != nullptr) sc = *sc_dev;  // scalars of a graph-replayed step
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        const int len = u.len;
        const int64_t k0 = u.shard_pos;
        // peel to an index that is a multiple of 8 (bf16 16-byte vectors)
        int head = (int)((8 - (k0 & 7)) & 7);
        if (head > len) head = len;
        const int nvec = (len - head) >> 3;
        const int done = head + 8 * nvec;
        if (u.is_pad) {
            const float zero8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if ((int)threadIdx.x < head) fused1(o, k0 + threadIdx.x, 0.0f, true, sc);
#pragma unroll 1
            for (int q = threadIdx.x; q < nvec; q += blockDim.x) {
                const int64_t k = k0 + head + 8 * (int64_t)q;
                float4 P[2], M[2], V[2];
                load_pmv8(o, k, P, M, V);
                fused8(o, k, zero8, P, M, V, true, sc);
            }
            if ((int)threadIdx.x < len - done) fused1(o, k0 + done + threadIdx.x, 0.0f, true, sc);
            continue;
        }
        const uint16_t* src_run = grads + u.arena_pos;
        if ((int)threadIdx.x < head)
            fused1(o, k0 + threadIdx.x,
                   finish(fold_scalar<NR>(src_run + threadIdx.x, stride, N), avg, fN), false, sc);
        // every rank's arena starts on a 16-byte boundary, so one phase D
        // holds for all N source streams
        const int D = bf16_phase(src_run + head);
        const uint16_t* src_al = src_run + head - D;
        if (D == 0) fused_body<NR, false>(src_al, stride, N, 0, o, k0 + head, nvec, avg, fN, sc);
        else fused_body<NR, true>(src_al, stride, N, D, o, k0 + head, nvec, avg, fN, sc);
        if ((int)threadIdx.x < len - done)
            fused1(o, k0 + done + threadIdx.x,
                   finish(fold_scalar<NR>(src_run + done + threadIdx.x, stride, N), avg, fN),
                   false, sc);
    }
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
             int op_avg) {
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
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

// ---------------------------------------------------------------------------
// FP8 (E4M3) all-gather copy-in and copy-out
//   amax_i = max |x| over parameter i (NaN ignored), scale_i = 448 / max(amax_i,
//   1e-12), ag8[k] = e4m3_rn(clamp(x * scale_i, -448, 448)), pads 0x00.
// ---------------------------------------------------------------------------

// Max |x| of each real unit, folded into its parameter's slot with an integer
// atomicMax (non-negative floats order like their bit patterns).
__global__ void __launch_bounds__(kThreads)
k_fp8_amax(const float* __restrict__ master, unsigned* __restrict__ amax_bits,
           const Unit* __restrict__ units, const int32_t* __restrict__ unit_param,
           int64_t n_real) {
    __shared__ float part[kThreads / 32];
    for (int64_t ui = blockIdx.x; ui < n_real; ui += gridDim.x) {
        const Unit u = units[ui];
        const float* src = master + u.shard_pos;
        const int len = u.len;
        const int head = (int)head_to_16B(src, len);
        float mx = 0.0f;
        for (int e = threadIdx.x; e < head; e += blockDim.x) mx = fmaxf(mx, fabsf(src[e]));
        const int nv = (len - head) >> 2;
        const float4* s4 = reinterpret_cast<const float4*>(src + head);
#pragma unroll 4
        for (int q = threadIdx.x; q < nv; q += blockDim.x) {
            const float4 x = __ldcs(s4 + q);
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
        }
        for (int e = head + 4 * nv + threadIdx.x; e < len; e += blockDim.x)
            mx = fmaxf(mx, fabsf(src[e]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = mx;
        __syncthreads();
        if (threadIdx.x < 32) {
            mx = threadIdx.x < kThreads / 32 ? part[threadIdx.x] : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (threadIdx.x == 0) atomicMax(amax_bits + unit_param[ui], __float_as_uint(mx));
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kThreads)
k_fp8_scales(float* __restrict__ scales, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) scales[i] = __fdiv_rn(448.0f, fmaxf(scales[i], 1e-12f));
}

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

__device__ __forceinline__ void zero_u8_run(uint8_t* __restrict__ dst, int len) {
    const int head = (int)head_to_16B(dst, len);
    if ((int)threadIdx.x < head) dst[threadIdx.x] = 0;
    const int nv = (len - head) >> 4;
    uint4* d = reinterpret_cast<uint4*>(dst + head);
    for (int q = threadIdx.x; q < nv; q += blockDim.x) __stcs(d + q, make_uint4(0u, 0u, 0u, 0u));
    const int done = head + 16 * nv;
    if ((int)threadIdx.x < len - done) dst[done + threadIdx.x] = 0;
}

__global__ void __launch_bounds__(kThreads, 4)
k_fp8_copy_in(const float* __restrict__ master, uint8_t* __restrict__ ag8,
              const float* __restrict__ scales, const Unit* __restrict__ units,
              const int32_t* __restrict__ unit_param, int64_t n_units) {
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        uint8_t* dst = ag8 + u.shard_pos;
        const int len = u.len;
        if (u.is_pad) {
            zero_u8_run(dst, len);
            continue;
        }
        const float sc = scales[unit_param[ui]];
        const float* src = master + u.shard_pos;
        // 16-byte output vectors; the fp32 source of a vector is then 64-byte aligned
        const int head = (int)head_to_16B(dst, len);
        if ((int)threadIdx.x < head) dst[threadIdx.x] = e4m3(fp8_in(src[threadIdx.x], sc));
        const int nv = (len - head) >> 4;
        const float4* s4 = reinterpret_cast<const float4*>(src + head);
        uint4* d = reinterpret_cast<uint4*>(dst + head);
#pragma unroll 1
        for (int q = threadIdx.x; q < nv; q += blockDim.x) {
            float4 x[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) x[k] = __ldcs(s4 + 4 * q + k);
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t lo = e4m3x2(fp8_in(x[k].x, sc), fp8_in(x[k].y, sc));
                const uint32_t hi = e4m3x2(fp8_in(x[k].z, sc), fp8_in(x[k].w, sc));
                w[k] = (lo & 0xFFFFu) | (hi << 16);
            }
            __stcs(d + q, make_uint4(w[0], w[1], w[2], w[3]));
        }
        const int done = head + 16 * nv;
        if ((int)threadIdx.x < len - done)
            dst[done + threadIdx.x] = e4m3(fp8_in(src[done + threadIdx.x], sc));
    }
}

// The 16 bytes that start D (1..15) bytes into the 32 bytes a:b.
__device__ __forceinline__ uint4 shift_bytes16(const uint4& a, const uint4& b, int D) {
    const int s = D >> 2;
    const uint32_t sh = 8u * (uint32_t)(D & 3);
    const uint32_t w0 = s == 0 ? a.x : s == 1 ? a.y : s == 2 ? a.z : a.w;
    const uint32_t w1 = s == 0 ? a.y : s == 1 ? a.z : s == 2 ? a.w : b.x;
    const uint32_t w2 = s == 0 ? a.z : s == 1 ? a.w : s == 2 ? b.x : b.y;
    const uint32_t w3 = s == 0 ? a.w : s == 1 ? b.x : s == 2 ? b.y : b.z;
    const uint32_t w4 = s == 0 ? b.x : s == 1 ? b.y : s == 2 ? b.z : b.w;
    return make_uint4(__funnelshift_r(w0, w1, sh), __funnelshift_r(w1, w2, sh),
                      __funnelshift_r(w2, w3, sh), __funnelshift_r(w3, w4, sh));
}

__global__ void __launch_bounds__(kThreads, 5)
k_fp8_copy_out(const uint8_t* __restrict__ ag8, uint8_t* __restrict__ arena8,
               const Unit* __restrict__ units, int64_t n_units) {
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        const int len = u.len;
        uint8_t* dst = arena8 + u.arena_pos;
        const uint8_t* src = ag8 + u.shard_pos;
        const int head = (int)head_to_16B(dst, len);
        if ((int)threadIdx.x < head) dst[threadIdx.x] = src[threadIdx.x];
        const int nv = (len - head) >> 4;
        const int D = (int)(reinterpret_cast<uintptr_t>(src + head) & 15u);
        const uint4* sa = reinterpret_cast<const uint4*>(src + head - D);
        uint4* d = reinterpret_cast<uint4*>(dst + head);
        if (D == 0) {
#pragma unroll 4
            for (int q = threadIdx.x; q < nv; q += blockDim.x) __stcs(d + q, __ldcs(sa + q));
        } else {
#pragma unroll 2
            for (int q = threadIdx.x; q < nv; q += blockDim.x)
                __stcs(d + q, shift_bytes16(__ldg(sa + q), __ldg(sa + q + 1), D));
        }
        const int done = head + 16 * nv;
        if ((int)threadIdx.x < len - done) dst[done + threadIdx.x] = src[done + threadIdx.x];
    }
}

// ---------------------------------------------------------------------------
// launch geometry
// ---------------------------------------------------------------------------

// One CTA per work item (tile, unit or chunk), launched in order.  On B200 a
// grid that covers the work once streams 12-17 % faster than a persistent
// grid-stride loop with a static cyclic assignment: the hardware hands out
// CTAs in index order as slots free up, so the addresses in flight stay a
// compact window instead of drifting apart across the arrays.
unsigned grid_for(const fsdp_group&, const void*, int64_t items) {
    return (unsigned)std::min<int64_t>(std::max<int64_t>(items, 1), 0x7FFFFFFF);
}

template <int NR>
cudaError_t launch_reduce_nr(const fsdp_group& g, const uint16_t* grads, int64_t stride, int N,
                             float* out, int64_t y_src_step, int64_t y_dst_step,
                             unsigned ydim, const Unit* units, int64_t n_units, int avg,
                             cudaStream_t st) {
    const void* kfn = (const void*)k_reduce_units<NR>;
    dim3 grid(grid_for(g, kfn, n_units), ydim);
    k_reduce_units<NR><<<grid, kThreads, 0, st>>>(grads, stride, N, out, y_src_step,
                                                  y_dst_step, units, n_units, avg);
    return cudaGetLastError();
}

template <int NR>
cudaError_t launch_rs_adamw_nr(const fsdp_group& g, const uint16_t* grads, const FusedOut& o,
                               int avg, const AdamScalars& sc, const AdamScalars* sc_dev,
                               cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    k_rs_adamw<NR><<<grid_for(g, (const void*)k_rs_adamw<NR>, nu), kThreads, 0, st>>>(
        grads, g.P_arena, g.N, o, g.d_units, nu, avg, sc, sc_dev);
    return cudaGetLastError();
}

// One thread: advance the device step counter and compute that step's AdamW
// scalars in binary64, in the same operation order as the host path.
__global__ void k_adamw_prepare(double lr, double beta1, double beta2, double eps, double wd,
                                int64_t* __restrict__ step, AdamScalars* __restrict__ out) {
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    const int64_t t = *step + 1;
    *step = t;
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
    *out = sc;
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

cudaError_t launch_copy_in(const fsdp_group& g, const float* master, uint16_t* ag,
                           cudaStream_t st) {
    const int64_t count = (int64_t)g.N * g.S;
    if (count == 0) return cudaSuccess;
    const bool pads = !g.tile_ranges.empty();
    k_copy_in<<<grid_for(g, (const void*)k_copy_in, g.n_tiles), kThreads, 0, st>>>(
        master, ag, count, g.n_tiles, pads ? g.d_intervals : nullptr,
        pads ? g.d_tile_ranges : nullptr);
    return cudaGetLastError();
}

cudaError_t launch_copy_out(const fsdp_group& g, const uint16_t* ag, uint16_t* arena,
                            cudaStream_t st) {
    if (g.n_real_units == 0) return cudaSuccess;
    k_copy_out<<<grid_for(g, (const void*)k_copy_out, g.n_real_units), kThreads, 0, st>>>(
        ag, arena, g.d_units, g.n_real_units);
    return cudaGetLastError();
}

cudaError_t launch_rs_fused(const fsdp_group& g, const uint16_t* grads, int op, float* reduced,
                            cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    if (nu == 0) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    const int64_t stride = g.P_arena;
    switch (g.N) {
#define FSDPK_CASE(K) \
    case K: return launch_reduce_nr<K>(g, grads, stride, g.N, reduced, 0, 0, 1, g.d_units, nu, avg, st);
        FSDPK_CASE(1) FSDPK_CASE(2) FSDPK_CASE(3) FSDPK_CASE(4)
        FSDPK_CASE(5) FSDPK_CASE(6) FSDPK_CASE(7) FSDPK_CASE(8)
#undef FSDPK_CASE
        default:
            return launch_reduce_nr<0>(g, grads, stride, g.N, reduced, 0, 0, 1, g.d_units, nu, avg,
                                       st);
    }
}

cudaError_t launch_rs_fused_units(int sm_count, int N, int64_t P_arena, const Unit* units,
                                  int64_t n_units, const uint16_t* grads, int op, float* reduced,
                                  cudaStream_t st) {
    if (n_units == 0) return cudaSuccess;
    fsdp_group g;  // only the SM count is read when sizing the grid
    g.sm_count = sm_count;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    switch (N) {
#define FSDPK_CASE(K) \
    case K: return launch_reduce_nr<K>(g, grads, P_arena, N, reduced, 0, 0, 1, units, n_units, avg, st);
        FSDPK_CASE(1) FSDPK_CASE(2) FSDPK_CASE(3) FSDPK_CASE(4)
        FSDPK_CASE(5) FSDPK_CASE(6) FSDPK_CASE(7) FSDPK_CASE(8)
#undef FSDPK_CASE
        default:
            return launch_reduce_nr<0>(g, grads, P_arena, N, reduced, 0, 0, 1, units, n_units, avg,
                                       st);
    }
}

cudaError_t launch_rs_pack(const fsdp_group& g, const uint16_t* grads, float* packed,
                           cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    if (nu == 0) return cudaSuccess;
    // blockIdx.y = source rank r: reads rank r's arena, writes packed[r]
    return launch_reduce_nr<1>(g, grads, 0, 1, packed, g.P_arena, (int64_t)g.N * g.S,
                               (unsigned)g.N, g.d_units, nu, 0, st);
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

cudaError_t launch_adamw(const fsdp_group& g, float* master, float* m, float* v,
                         const float* grad, const AdamScalars& sc, cudaStream_t st,
                         const AdamScalars* sc_dev) {
    const int64_t count = (int64_t)g.N * g.S;
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

cudaError_t launch_shard(const fsdp_group& g, const float* full, float* master,
                         cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    if (nu == 0) return cudaSuccess;
    k_shard<<<grid_for(g, (const void*)k_shard, nu), kThreads, 0, st>>>(full, master, g.d_units,
                                                                        nu);
    return cudaGetLastError();
}

}  // namespace fsdpk

namespace fsdpk {

cudaError_t launch_rs_adamw(const fsdp_group& g, const uint16_t* grads, int op, float* master,
                            float* m, float* v, const AdamScalars& sc, uint16_t* ag_next,
                            float* reduced, cudaStream_t st, const AdamScalars* sc_dev) {
    if (g.units.empty()) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    const FusedOut o{master, m, v, reduced, ag_next};
    switch (g.N) {
#define FSDPK_CASE(K) \
    case K: return launch_rs_adamw_nr<K>(g, grads, o, avg, sc, sc_dev, st);
        FSDPK_CASE(1) FSDPK_CASE(2) FSDPK_CASE(3) FSDPK_CASE(4)
        FSDPK_CASE(5) FSDPK_CASE(6) FSDPK_CASE(7) FSDPK_CASE(8)
#undef FSDPK_CASE
        default:
            return launch_rs_adamw_nr<0>(g, grads, o, avg, sc, sc_dev, st);
    }
}

}  // namespace fsdpk

namespace fsdpk {

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
            acc, grads, g.P_arena, g.N, reduced, g.d_units, nu, avg);
    else
        k_reduce_acc<false><<<grid_for(g, (const void*)k_reduce_acc<false>, nu), kThreads, 0, st>>>(
            acc, grads, g.P_arena, g.N, reduced, g.d_units, nu, avg);
    return cudaGetLastError();
}

}  // namespace fsdpk

namespace fsdpk {

cudaError_t launch_copy_in_fp8(const fsdp_group& g, const float* master, uint8_t* ag8,
                               float* scales, cudaStream_t st) {
    if (g.n > 0) {
        cudaError_t e = cudaMemsetAsync(scales, 0, (size_t)g.n * sizeof(float), st);
        if (e != cudaSuccess) return e;
        if (g.n_real_units > 0)
            k_fp8_amax<<<grid_for(g, nullptr, g.n_real_units), kThreads, 0, st>>>(
                master, reinterpret_cast<unsigned*>(scales), g.d_units, g.d_unit_param,
                g.n_real_units);
        k_fp8_scales<<<(unsigned)((g.n + kThreads - 1) / kThreads), kThreads, 0, st>>>(scales, g.n);
    }
    const int64_t nu = (int64_t)g.units.size();
    if (nu > 0)
        k_fp8_copy_in<<<grid_for(g, nullptr, nu), kThreads, 0, st>>>(master, ag8, scales,
                                                                     g.d_units, g.d_unit_param, nu);
    return cudaGetLastError();
}

cudaError_t launch_copy_out_fp8(const fsdp_group& g, const uint8_t* ag8, uint8_t* arena8,
                                cudaStream_t st) {
    if (g.n_real_units == 0) return cudaSuccess;
    k_fp8_copy_out<<<grid_for(g, nullptr, g.n_real_units), kThreads, 0, st>>>(ag8, arena8,
                                                                              g.d_units,
                                                                              g.n_real_units);
    return cudaGetLastError();
}

}  // namespace fsdpk
