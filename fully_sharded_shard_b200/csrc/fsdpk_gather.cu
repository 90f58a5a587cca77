// fsdpk_gather.cu -- the all-gather half of the step and the set-up shard:
// copy-in (fp32 shards -> bf16 slots of the rank-major all-gather buffer),
// copy-out (the buffer -> unsharded per-parameter views), Shard(0)
// placement, and the FP8 (E4M3) copy-in / copy-out.
//   copy-in  -- "Sharded Training: FSDP2, DTensor, Tensor and Pipeline
//               Parallelism", Mixed precision paragraph: bf16 copies of the fp32
//               shards are all-gathered.
//   copy-out -- "Introduction to PyTorch FSDP2 Backend Features", Working
//               Principle (All-Gather state): shards become full parameters.
//   FP8      -- "PyTorch FSDP2 Guide: Distributed LLM Training with DTensor",
//               Deep Dive, 2. Native FP8 Training with Float8Tensor.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cuda_fp8.h>

#include "fsdpk_device.cuh"

namespace fsdpk {
namespace {

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
          const TileRange* __restrict__ tr FSDPK_DBG_PARAM) {
    for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x) {
        const int64_t base = t * kCopyInTile;
        const int64_t end = min(base + kCopyInTile, count);
        TileRange rng{0, 0};
        if (tr != nullptr) rng = tr[t];
        FSDPK_GUARD(end <= dbg.ns && rng.begin >= 0 && rng.begin <= rng.end &&
                        rng.end <= dbg.n_aux, t);
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
// copy-out: arena[arena_pos + e] = ag[shard_pos + e] for each real unit
// ---------------------------------------------------------------------------
// The destination of a unit is peeled to a 16-byte boundary; its source then
// sits at a phase D (in elements) inside its 16-byte vectors, the same for
// the whole unit.  A misaligned source is read once, in aligned 16-byte
// vectors: a team of NW warps covers NW x 128 consecutive vectors per pass,
// warp w's lanes holding vectors w*128 + 32k + lane (k = 0..3), and each
// output vector takes its upper half from the next source vector, which the
// next lane holds (one shuffle per 32-bit word); the last lane takes it from
// lane 0's next slot, or from one extra load after the last slot.
// Long units get a CTA (a team of 8 warps) each; short units are packed, a
// warp per unit, so that a group of many small parameters does not pay a
// CTA launch per run.

__device__ __forceinline__ uint4 shfl_next(const uint4& v, int src) {
    uint4 r;
    r.x = __shfl_sync(0xffffffffu, v.x, src);
    r.y = __shfl_sync(0xffffffffu, v.y, src);
    r.z = __shfl_sync(0xffffffffu, v.z, src);
    r.w = __shfl_sync(0xffffffffu, v.w, src);
    return r;
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

// One unit by a team of NW warps (this thread is lane `lane` of warp w of
// the team, index t = 32 w + lane), in one pass: the team's 4 x 32 x NW
// slots cover every 16-byte vector of the unit after the destination's head
// peel (a long unit has at most kUnitElems elements, a short one fewer than
// kShortRun).  T = uint16_t (bf16) or uint8_t.
template <int NW, typename T>
__device__ __forceinline__ void copy_unit(const T* src_run, T* dst_run, int len, int w, int lane,
                                          int t) {
    constexpr int kVec = 16 / (int)sizeof(T);
    static_assert(kUnitElems <= 8 * 128 * 8 && kShortRun <= 128 * 8, "one pass per unit");
    const int head = (int)head_to_16B(dst_run, len);
    if (t < head) dst_run[t] = src_run[t];
    const int nvec = (len - head) / kVec;
    const int D = (int)((reinterpret_cast<uintptr_t>(src_run + head) / sizeof(T)) & (kVec - 1));
    const uint4* s = reinterpret_cast<const uint4*>(src_run + head - D);
    uint4* d = reinterpret_cast<uint4*>(dst_run + head);
    const int q0 = w * 128;
    // a misaligned run also reads vector nvec, which holds its last elements
    const int lim = D ? nvec : nvec - 1;
    uint4 a[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int q = q0 + 32 * k + lane;
        if (nvec > 0 && q <= lim) a[k] = __ldcs(s + q);
    }
    uint4 e = a[0];
    if (NW > 1 && D != 0 && lane == 0 && q0 + 128 <= nvec) e = __ldcs(s + q0 + 128);
    const int nxt = (lane + 1) & 31;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int q = q0 + 32 * k + lane;
        uint4 o = a[k];
        if (D != 0) {  // uniform across the team
            // lane l takes lane l+1's vector; lane 31 takes the first vector of
            // the next 32, which lane 0 holds (its next slot, or e after the last)
            const uint4 b = shfl_next(lane == 0 ? (k < 3 ? a[k < 3 ? k + 1 : 0] : e) : a[k], nxt);
            if constexpr (sizeof(T) == 2) o = shift_bf16x8(a[k], b, D);
            else o = shift_bytes16(a[k], b, D);
        }
        if (q < nvec) __stcs(d + q, o);
    }
    const int done = head + kVec * nvec;
    if (t < len - done) dst_run[done + t] = src_run[done + t];
}

// CTAs [0, n_packs) copy one pack of short units each, a warp per unit; the
// others one long unit each (a team of 8 warps).  One launch, so the packs
// are not a second, small grid that waits for SM slots behind another
// stream's kernel; and first in it, so that their CTAs -- a few dependent
// round trips per warp -- run beside the long units rather than after them.
// TAB: unit ui's rows come from unit_src[ui] (a pull from wherever that
// rank's slot lives, resolved on the host), instead of ag + shard_pos.
// A pack of short units, a warp per unit: not inlined into k_copy_out, so
// that its registers do not add to those of the long-unit path.
template <bool TAB, typename T>
__device__ __noinline__ void copy_out_pack(const T* __restrict__ ag,
                                           const T* const* __restrict__ unit_src,
                                           T* __restrict__ arena, const Unit* __restrict__ units,
                                           int b, int e FSDPK_DBG_PARAM) {
    const int lane = threadIdx.x & 31;
    for (int ui = b + (int)(threadIdx.x >> 5); ui < e; ui += kThreads / 32) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, TAB ? kChkArena : (kChkShard | kChkArena));
        const T* src = TAB ? unit_src[ui] : ag + u.shard_pos;
        copy_unit<1>(src, arena + u.arena_pos, u.len, 0, lane, lane);
    }
}

template <bool TAB, typename T>
__global__ void __launch_bounds__(kThreads, 5)
k_copy_out(const T* __restrict__ ag, const T* const* __restrict__ unit_src,
           T* __restrict__ arena, const Unit* __restrict__ units, int64_t n_packs,
           const int32_t* __restrict__ packs FSDPK_DBG_PARAM) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if ((int64_t)blockIdx.x >= n_packs) {
        const int64_t ui = (int64_t)blockIdx.x - n_packs;  // long units are units [0, n_long)
        const Unit u = units[ui];
#ifdef FSDPK_DEBUG
        // a pulled unit's source is a pointer of the table, not a shard position
        if (!unit_in_bounds(dbg, u, ui, TAB ? kChkArena : (kChkShard | kChkArena))) return;
#endif
        const T* src = TAB ? unit_src[ui] : ag + u.shard_pos;
        copy_unit<kThreads / 32>(src, arena + u.arena_pos, u.len, warp, lane, threadIdx.x);
        return;
    }
    const int p = (int)blockIdx.x;
    copy_out_pack<TAB>(ag, unit_src, arena, units, packs[p], packs[p + 1] FSDPK_DBG_ARG(dbg));
}

// The copy-out of a plan's real units: the long ones and the packs.
template <bool TAB, typename T>
cudaError_t launch_copy_out_units(const fsdp_group& g, const T* ag, const T* const* unit_src,
                                  T* arena, int32_t dbg_kernel, cudaStream_t st) {
    (void)dbg_kernel;
    const int64_t n_packs = (int64_t)g.packs.size() - 1;
    k_copy_out<TAB, T><<<grid_for(g, nullptr, n_packs + g.n_long_units), kThreads, 0, st>>>(
        ag, unit_src, arena, g.d_units, n_packs, g.d_packs
        FSDPK_DBG_ARG(debug_bounds(g, dbg_kernel)));
    return cudaGetLastError();
}

// Flat copy-out (a group of many small parameters): one CTA per tile of
// kFlatTile elements of the arena, kFlatV vectors of 8 per thread with their
// codes read first.  A vector inside one real run takes its 8 elements from
// the aligned 16-byte vectors of the buffer that hold them (shifted by the
// run's phase) in one 16-byte store, every vector's loads issued before the
// stores; a gap vector is left alone.  Mixed vectors go a thread per
// element.
// One launch: CTAs [0, mixed_ctas) take the mixed vectors' elements,
// kFlatMixedPer a thread (element t + i * T, T the region's threads, is
// element e = t % 8 of list entry m = t / 8: arena element k = 8 * mixq[m] + e
// with code mixc[t]; gaps untouched), first in the grid; the others one tile
// each.
__global__ void __launch_bounds__(kThreads)
k_copy_out_flat(const uint16_t* __restrict__ ag, uint16_t* __restrict__ arena, int64_t count,
                const int32_t* __restrict__ amap, const int32_t* __restrict__ mixq,
                const int32_t* __restrict__ mixc, int64_t n_mixed, int64_t mixed_ctas
                FSDPK_DBG_PARAM) {
    if ((int64_t)blockIdx.x < mixed_ctas) {
        const int64_t t0 = (int64_t)blockIdx.x * kThreads + threadIdx.x, T = mixed_ctas * kThreads;
        int64_t k[kFlatMixedPer];
        uint16_t x[kFlatMixedPer];
        bool on[kFlatMixedPer];
#pragma unroll
        for (int i = 0; i < kFlatMixedPer; ++i) {
            const int64_t t = t0 + i * T;
            on[i] = t < 8 * n_mixed;
            k[i] = on[i] ? 8 * (int64_t)mixq[t >> 3] + (t & 7) : 0;
            const int32_t c = on[i] ? mixc[t] : kFlatPad;
            const int64_t src = k[i] + (c >> 1);
            on[i] = on[i] && k[i] < count && c != kFlatPad;
#ifdef FSDPK_DEBUG
            if (on[i] && !debug_ok_thread(dbg, k[i] < dbg.arena && src >= 0 && src < dbg.ns, k[i]))
                on[i] = false;
#endif
            if (on[i]) x[i] = ag[src];
        }
#pragma unroll
        for (int i = 0; i < kFlatMixedPer; ++i)
            if (on[i]) arena[k[i]] = x[i];
        return;
    }
    const int64_t nv = (count + 7) >> 3;
    const int64_t q0 = ((int64_t)blockIdx.x - mixed_ctas) * (kThreads * kFlatV) + threadIdx.x;
    int32_t code[kFlatV];
    flat_tile_codes(amap, q0, nv, code);
    uint4 x[kFlatV], y[kFlatV];
    int D[kFlatV];
#pragma unroll
    for (int j = 0; j < kFlatV; ++j) {
        const int64_t k = 8 * (q0 + (int64_t)j * kThreads);
        const int32_t c = code[j];
        D[j] = 0;
        if (!(c & 1) && c != kFlatPad) {
            const int64_t src = k + (c >> 1);
#ifdef FSDPK_DEBUG
            if (!debug_ok_thread(dbg, k + 8 <= count && k + 8 <= dbg.arena && src >= 0 &&
                                          src + 8 <= dbg.ns, k)) {
                code[j] = kFlatPad;
                continue;
            }
#endif
            D[j] = (int)(src & 7);
            const uint4* s = reinterpret_cast<const uint4*>(ag + (src - D[j]));
            x[j] = __ldg(s);
            if (D[j] != 0) y[j] = __ldg(s + 1);
            else y[j] = x[j];
        }
    }
#pragma unroll
    for (int j = 0; j < kFlatV; ++j) {
        const int32_t c = code[j];
        if (!(c & 1) && c != kFlatPad)
            __stcs(reinterpret_cast<uint4*>(arena + 8 * (q0 + (int64_t)j * kThreads)),
                   shift_bf16x8(x[j], y[j], D[j]));
    }
}

// ---------------------------------------------------------------------------
// shard: master[shard_pos + e] = full[arena_pos + e]; pads +0 (set-up path)
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kThreads)
k_shard(const float* __restrict__ full, float* __restrict__ master,
        const Unit* __restrict__ units, int64_t n_units FSDPK_DBG_PARAM) {
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard | kChkArena);
        if (u.is_pad) {
            zero_f32_run(master + u.shard_pos, u.len);
            continue;
        }
        for (int64_t e = threadIdx.x; e < u.len; e += blockDim.x)
            master[u.shard_pos + e] = full[u.arena_pos + e];
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
           int64_t n_real FSDPK_DBG_PARAM) {
    __shared__ float part[kThreads / 32];
    for (int64_t ui = blockIdx.x; ui < n_real; ui += gridDim.x) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard);
        FSDPK_GUARD(unit_param[ui] >= 0 && unit_param[ui] < dbg.n_aux, ui);
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
              const int32_t* __restrict__ unit_param, int64_t n_units FSDPK_DBG_PARAM) {
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard);
        FSDPK_GUARD(u.is_pad || (unit_param[ui] >= 0 && unit_param[ui] < dbg.n_aux), ui);
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

// scales[i] = 448 / max(max over the D devices of amax_d[i], 1e-12): the
// per-parameter amax is the maximum of the devices' partial maxima (each
// device saw only its own ranks' rows).
__global__ void __launch_bounds__(kThreads)
k_fp8_scales_from_parts(const unsigned* const* __restrict__ amax_tab, int D,
                        float* __restrict__ scales, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float mx = 0.0f;
    for (int d = 0; d < D; ++d) mx = fmaxf(mx, __uint_as_float(amax_tab[d][i]));
    scales[i] = __fdiv_rn(448.0f, fmaxf(mx, 1e-12f));
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

cudaError_t launch_copy_in(const fsdp_group& g, const float* master, uint16_t* ag,
                           cudaStream_t st) {
    const int64_t count = (int64_t)g.L * g.S;
    if (count == 0) return cudaSuccess;
    const bool pads = !g.tile_ranges.empty();
    k_copy_in<<<grid_for(g, (const void*)k_copy_in, g.n_tiles), kThreads, 0, st>>>(
        master, ag, count, g.n_tiles, pads ? g.d_intervals : nullptr,
        pads ? g.d_tile_ranges : nullptr
        FSDPK_DBG_ARG(debug_bounds(g, kDbgCopyIn, (int64_t)g.intervals.size())));
    return cudaGetLastError();
}

cudaError_t launch_copy_out(const fsdp_group& g, const uint16_t* ag, uint16_t* arena,
                            cudaStream_t st) {
    if (g.n_real_units == 0) return cudaSuccess;
    if (g.flat_copy_out) {
        const int64_t n_mixed = (int64_t)g.amixq.size();
        const int64_t mixed_ctas = flat_mixed_ctas(n_mixed);
        k_copy_out_flat<<<(unsigned)(flat_grid(g.P_arena) + mixed_ctas), kThreads, 0, st>>>(
            ag, arena, g.P_arena, g.d_amap, g.d_amixq, g.d_amixc, n_mixed, mixed_ctas
            FSDPK_DBG_ARG(debug_bounds(g, kDbgCopyOutFlat)));
        return cudaGetLastError();
    }
    return launch_copy_out_units<false, uint16_t>(g, ag, nullptr, arena, kDbgCopyOut, st);
}

cudaError_t launch_copy_out_tab(const fsdp_group& parent, const uint16_t* const* unit_src,
                                uint16_t* arena, cudaStream_t st) {
    if (parent.n_real_units == 0) return cudaSuccess;
    return launch_copy_out_units<true, uint16_t>(parent, nullptr, unit_src, arena,
                                                 kDbgCopyOutTab, st);
}

cudaError_t launch_shard(const fsdp_group& g, const float* full, float* master,
                         cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    if (nu == 0) return cudaSuccess;
    k_shard<<<grid_for(g, (const void*)k_shard, nu), kThreads, 0, st>>>(
        full, master, g.d_units, nu FSDPK_DBG_ARG(debug_bounds(g, kDbgShard)));
    return cudaGetLastError();
}

cudaError_t launch_copy_in_fp8(const fsdp_group& g, const float* master, uint8_t* ag8,
                               float* scales, cudaStream_t st) {
    if (g.n > 0) {
        cudaError_t e = cudaMemsetAsync(scales, 0, (size_t)g.n * sizeof(float), st);
        if (e != cudaSuccess) return e;
        if (g.n_real_units > 0)
            k_fp8_amax<<<grid_for(g, nullptr, g.n_real_units), kThreads, 0, st>>>(
                master, reinterpret_cast<unsigned*>(scales), g.d_units, g.d_unit_param,
                g.n_real_units FSDPK_DBG_ARG(debug_bounds(g, kDbgFp8Amax, g.n)));
        k_fp8_scales<<<(unsigned)((g.n + kThreads - 1) / kThreads), kThreads, 0, st>>>(scales, g.n);
    }
    const int64_t nu = (int64_t)g.units.size();
    if (nu > 0)
        k_fp8_copy_in<<<grid_for(g, nullptr, nu), kThreads, 0, st>>>(
            master, ag8, scales, g.d_units, g.d_unit_param, nu
            FSDPK_DBG_ARG(debug_bounds(g, kDbgFp8CopyIn, g.n)));
    return cudaGetLastError();
}

cudaError_t launch_fp8_scales_from_amax(const fsdp_group& g, float* scales, cudaStream_t st) {
    if (g.n == 0) return cudaSuccess;
    k_fp8_scales<<<(unsigned)((g.n + kThreads - 1) / kThreads), kThreads, 0, st>>>(scales, g.n);
    return cudaGetLastError();
}

cudaError_t launch_copy_in_fp8_scaled(const fsdp_group& g, const float* master, uint8_t* ag8,
                                      const float* scales, cudaStream_t st) {
    const int64_t nu = (int64_t)g.units.size();
    if (nu > 0)
        k_fp8_copy_in<<<grid_for(g, nullptr, nu), kThreads, 0, st>>>(
            master, ag8, scales, g.d_units, g.d_unit_param, nu
            FSDPK_DBG_ARG(debug_bounds(g, kDbgFp8CopyIn, g.n)));
    return cudaGetLastError();
}

cudaError_t launch_copy_out_fp8(const fsdp_group& g, const uint8_t* ag8, uint8_t* arena8,
                                cudaStream_t st) {
    if (g.n_real_units == 0) return cudaSuccess;
    return launch_copy_out_units<false, uint8_t>(g, ag8, nullptr, arena8, kDbgFp8CopyOut, st);
}

cudaError_t launch_copy_out_fp8_tab(const fsdp_group& parent, const uint8_t* const* unit_src,
                                    uint8_t* arena8, cudaStream_t st) {
    if (parent.n_real_units == 0) return cudaSuccess;
    return launch_copy_out_units<true, uint8_t>(parent, nullptr, unit_src, arena8,
                                                kDbgFp8CopyOutTab, st);
}

cudaError_t launch_fp8_scales_from_parts(const unsigned* const* amax_tab, int D, float* scales,
                                         int n, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    k_fp8_scales_from_parts<<<(unsigned)((n + kThreads - 1) / kThreads), kThreads, 0, st>>>(
        amax_tab, D, scales, n);
    return cudaGetLastError();
}

}  // namespace fsdpk
