// fsdpk_step.cu -- the whole step of one small parameter group in one launch.
//
// The step of one group is copy-in, copy-out, reduce-scatter and AdamW
// ("Introduction to PyTorch FSDP2 Backend Features", Working Principle).  A
// group of a few thousand elements (the two-layer MLP of the ZeroRedundancy-
// Optimizer paragraph of "Sharded Training: FSDP2, DTensor, Tensor and
// Pipeline Parallelism" has 676) moves a few kilobytes per stage, so four
// launches cost more than the data: here one CTA runs the four stages with a
// block barrier between dependent ones.  The per-element arithmetic is that of
// the four stage kernels, so the results are the same bits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fsdpk_device.cuh"

namespace fsdpk {
namespace {

constexpr int kStepThreads = 512;

// Shared memory holds the cast copy and the reduced gradient, so the stages
// hand them over without a round trip to global memory.
__global__ void __launch_bounds__(kStepThreads, 1)
k_small_step(float* __restrict__ p, float* __restrict__ m, float* __restrict__ v,
             const uint16_t* __restrict__ grads, int64_t P_arena, int N,
             uint16_t* __restrict__ ag, uint16_t* __restrict__ arena, float* __restrict__ red,
             const Unit* __restrict__ units, int64_t n_units, int64_t count, int op_avg,
             AdamScalars sc, const AdamScalars* __restrict__ sc_dev) {
    extern __shared__ float smem[];
    float* red_s = smem;                                            // [count]
    uint16_t* ag_s = reinterpret_cast<uint16_t*>(smem + count);     // [count]
    if (sc_dev != nullptr) sc = *sc_dev;  // scalars of a graph-replayed step
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    // one warp per work unit, its lanes over the unit's elements, so that the
    // units' memory accesses are in flight together; a warp keeps its first
    // unit in registers for the second stage
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int n_warps = blockDim.x >> 5;
    Unit first{};
    if (warp < n_units) first = units[warp];
    // copy-in: the units cover [N][S] (real rows cast, pad rows +0)
    for (int64_t ui = warp; ui < n_units; ui += n_warps) {
        const Unit u = ui == warp ? first : units[ui];
        for (int e = lane; e < u.len; e += 32) {
            const int64_t k = u.shard_pos + e;
            const __nv_bfloat16 h = __float2bfloat16_rn(u.is_pad ? 0.0f : p[k]);
            const uint16_t bits = *reinterpret_cast<const uint16_t*>(&h);
            ag[k] = bits;
            ag_s[k] = bits;
        }
    }
    __syncthreads();  // the copy-out reads what other warps cast
    // copy-out of the real rows and the rank-ordered reduce-scatter
    for (int64_t ui = warp; ui < n_units; ui += n_warps) {
        const Unit u = ui == warp ? first : units[ui];
        for (int e = lane; e < u.len; e += 32) {
            const int64_t k = u.shard_pos + e;
            float g = 0.0f;
            if (!u.is_pad) {
                arena[u.arena_pos + e] = ag_s[k];
                const uint16_t* src = grads + u.arena_pos + e;
                float acc = bf16_bits_to_f32(src[0]);
                for (int r = 1; r < N; ++r)
                    acc = __fadd_rn(acc, bf16_bits_to_f32(src[(int64_t)r * P_arena]));
                g = finish(acc, avg, fN);
            }
            red[k] = g;
            red_s[k] = g;
        }
    }
    __syncthreads();  // AdamW reads the reduced gradient of every rank
    for (int64_t k = threadIdx.x; k < count; k += blockDim.x) {
        float pp = p[k], mm = m[k], vv = v[k];
        adamw1(pp, mm, vv, red_s[k], sc);
        p[k] = pp;
        m[k] = mm;
        v[k] = vv;
    }
}

}  // namespace

cudaError_t launch_small_step(const fsdp_group& g, float* master, float* m, float* v,
                              const uint16_t* grads, int op, uint16_t* ag, uint16_t* arena,
                              float* reduced, const AdamScalars& sc, const AdamScalars* sc_dev,
                              cudaStream_t st) {
    const int64_t count = (int64_t)g.L * g.S;
    if (count == 0) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    // fp32 reduced gradient + bf16 copy per element: 6 * count bytes, within
    // the 48 KB of dynamic shared memory a launch gets without opting in
    const size_t smem = (size_t)count * (sizeof(float) + sizeof(uint16_t));
    k_small_step<<<1, kStepThreads, smem, st>>>(master, m, v, grads, g.P_arena, g.N, ag, arena,
                                                reduced, g.d_units, (int64_t)g.units.size(),
                                                count, avg, sc, sc_dev);
    return cudaGetLastError();
}

}  // namespace fsdpk
