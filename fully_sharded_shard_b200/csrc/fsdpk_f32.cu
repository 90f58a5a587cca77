// fsdpk_f32.cu -- the all-gather copy-in and copy-out with param_dtype fp32,
// a test mode: with no cast, all-gather(shard(x)) == x holds bit for bit, the
// identity the bf16 path can only meet up to rounding.
//   "Sharded Training: FSDP2, DTensor, Tensor and Pipeline Parallelism",
//   Mixed precision paragraph (MixedPrecisionPolicy param_dtype; fp32 when no
//   policy is given) and fully_shard paragraph (Shard(0), padded chunks).
#include <cuda_runtime.h>

#include <cstdint>

#include "fsdpk.h"
#include "fsdpk_device.cuh"

namespace fsdpk {
namespace {

// Copy `len` fp32 elements from src to dst (zeros when src is null), 16-byte
// vectors where both sides share their phase inside a 16-byte vector,
// element by element otherwise.
__device__ __forceinline__ void copy_f32_run(const float* __restrict__ src, float* __restrict__ dst,
                                             int64_t len) {
    const bool zero = src == nullptr;
    const int64_t head = head_to_16B(dst, len);
    const bool congruent =
        zero || ((reinterpret_cast<uintptr_t>(src) ^ reinterpret_cast<uintptr_t>(dst)) & 15u) == 0;
    if (!congruent) {
        for (int64_t e = threadIdx.x; e < len; e += blockDim.x) dst[e] = src[e];
        return;
    }
    if (threadIdx.x < head) dst[threadIdx.x] = zero ? 0.0f : src[threadIdx.x];
    const int64_t nv = (len - head) >> 2;
    float4* d4 = reinterpret_cast<float4*>(dst + head);
    const float4* s4 = zero ? nullptr : reinterpret_cast<const float4*>(src + head);
    for (int64_t q = threadIdx.x; q < nv; q += blockDim.x)
        __stcs(d4 + q, zero ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldcs(s4 + q));
    const int64_t done = head + 4 * nv;
    if (threadIdx.x < len - done) dst[done + threadIdx.x] = zero ? 0.0f : src[done + threadIdx.x];
}

// ag32[shard_pos + e] = master[shard_pos + e] on real units, +0 on pad units.
__global__ void __launch_bounds__(kThreads)
k_copy_in_f32(const float* __restrict__ master, float* __restrict__ ag32,
              const Unit* __restrict__ units, int64_t n_units FSDPK_DBG_PARAM) {
    for (int64_t ui = blockIdx.x; ui < n_units; ui += gridDim.x) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard);
        copy_f32_run(u.is_pad ? nullptr : master + u.shard_pos, ag32 + u.shard_pos, u.len);
    }
}

// arena32[arena_pos + e] = ag32[shard_pos + e] on real units.
__global__ void __launch_bounds__(kThreads)
k_copy_out_f32(const float* __restrict__ ag32, float* __restrict__ arena32,
               const Unit* __restrict__ units, int64_t n_real FSDPK_DBG_PARAM) {
    for (int64_t ui = blockIdx.x; ui < n_real; ui += gridDim.x) {
        const Unit u = units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard | kChkArena);
        copy_f32_run(ag32 + u.shard_pos, arena32 + u.arena_pos, u.len);
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int status_of(cudaError_t e) { return e == cudaSuccess ? FSDP_OK : record_cuda_error(e); }

}  // namespace
}  // namespace fsdpk

extern "C" {

int fsdp_copy_in_f32(fsdp_group_t g, const float* master, float* ag32, fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if ((int64_t)g->L * g->S > 0 && (master == nullptr || ag32 == nullptr)) return FSDP_EINVAL;
    if (!fsdpk::aligned16(master) || !fsdpk::aligned16(ag32)) return FSDP_EALIGN;
    int st = fsdpk::check_plan_device(g);
    if (st != FSDP_OK) return st;
    const int64_t nu = (int64_t)g->units.size();
    if (nu == 0) return FSDP_OK;
    fsdpk::k_copy_in_f32<<<fsdpk::grid_for(*g, nullptr, nu), fsdpk::kThreads, 0,
                           (cudaStream_t)stream>>>(master, ag32, g->d_units, nu
                           FSDPK_DBG_ARG(fsdpk::debug_bounds(*g, fsdpk::kDbgCopyInF32)));
    return fsdpk::status_of(cudaGetLastError());
}

int fsdp_copy_out_f32(fsdp_group_t g, const float* ag32, float* arena32, fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if (g->P > 0 && (ag32 == nullptr || arena32 == nullptr)) return FSDP_EINVAL;
    if (!fsdpk::aligned16(ag32) || !fsdpk::aligned16(arena32)) return FSDP_EALIGN;
    int st = fsdpk::check_plan_device(g);
    if (st != FSDP_OK) return st;
    if (g->n_real_units == 0) return FSDP_OK;
    fsdpk::k_copy_out_f32<<<fsdpk::grid_for(*g, nullptr, g->n_real_units), fsdpk::kThreads, 0,
                            (cudaStream_t)stream>>>(ag32, arena32, g->d_units, g->n_real_units
                            FSDPK_DBG_ARG(fsdpk::debug_bounds(*g, fsdpk::kDbgCopyOutF32)));
    return fsdpk::status_of(cudaGetLastError());
}

}  // extern "C"
