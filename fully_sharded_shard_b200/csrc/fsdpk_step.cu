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
constexpr int kStepPerThread = 16;  // AdamW elements per thread: 512 x 16 = 8192
constexpr int kSmallStepMaxRanks = 8;  // ranks whose gradients are loaded together
static_assert(kStepThreads * kStepPerThread == FSDP_SMALL_STEP_ELEMS, "small-step capacity");

// The step is bound by dependent memory round trips, not by bytes, so the
// kernel issues every load that does not depend on another one up front:
//   1. the thread's AdamW elements of master, m and v (registers), the
//      master also into shared memory for the copy-in, and the warp's first
//      work unit; then a block barrier;
//   2. per work unit (one warp each, lanes over its elements): the N ranks'
//      gradients of the unit's real rows, issued before the cast of the
//      master from shared memory; the copy-in, copy-out and rank-ordered
//      fold of an element all happen in the thread that owns it, so no
//      barrier separates them; the reduced gradient goes to shared memory;
//      then a block barrier;
//   3. AdamW on the registers of step 1 and the reduced gradient.
// Two dependent global round trips (the unit table and master / moments,
// then the gradients) instead of four.  Shared memory: the fp32 master, then
// in the same words the reduced gradient (each element is read and written
// by the one thread that owns it in step 2), 4 bytes per element.
__global__ void __launch_bounds__(kStepThreads, 1)
k_small_step(float* __restrict__ p, float* __restrict__ m, float* __restrict__ v,
             const uint16_t* __restrict__ grads, int64_t P_arena, int N,
             uint16_t* __restrict__ ag, uint16_t* __restrict__ arena, float* __restrict__ red,
             const Unit* __restrict__ units, int64_t n_units, int64_t count, int op_avg,
             AdamScalars sc, const AdamScalars* __restrict__ sc_dev, StepCounter ctr
             FSDPK_DBG_PARAM) {
    extern __shared__ float smem[];  // [count]: master, then the reduced gradient
    __shared__ AdamScalars s_sc;
    const bool avg = op_avg != 0;
    const float fN = (float)N;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int n_warps = blockDim.x >> 5;
    // step 1: every independent load
    Unit first{};
    if (warp < n_units) first = units[warp];
    if (sc_dev != nullptr) sc = *sc_dev;  // scalars of a graph-replayed step
    if (ctr.step != nullptr && threadIdx.x == 0) {
        // the step of a graph-replayed call: advance the device counter and
        // compute its scalars here (read after the block barrier below)
        const int64_t t = *ctr.step + 1;
        *ctr.step = t;
        s_sc = adam_scalars_dev(ctr.lr, ctr.beta1, ctr.beta2, ctr.eps, ctr.wd, t);
        if (ctr.out != nullptr) *ctr.out = s_sc;
    }
    float pp[kStepPerThread], mm[kStepPerThread], vv[kStepPerThread];
#pragma unroll
    for (int j = 0; j < kStepPerThread; ++j) {
        const int64_t k = threadIdx.x + (int64_t)j * kStepThreads;
        if (k < count) {
            pp[j] = p[k];
            mm[j] = m[k];
            vv[j] = v[k];
        }
    }
#pragma unroll
    for (int j = 0; j < kStepPerThread; ++j) {
        const int64_t k = threadIdx.x + (int64_t)j * kStepThreads;
        if (k < count) smem[k] = pp[j];
    }
    __syncthreads();
    if (ctr.step != nullptr) sc = s_sc;
    // step 2: per unit, the gradients first, then cast, copy out, fold
    for (int64_t ui = warp; ui < n_units; ui += n_warps) {
        const Unit u = ui == warp ? first : units[ui];
        FSDPK_UNIT_GUARD(u, ui, kChkShard | kChkArena);
#pragma unroll 2
        for (int e = lane; e < u.len; e += 32) {
            const int64_t k = u.shard_pos + e;
            if (u.is_pad) {
                ag[k] = 0;  // +0 in pad rows
                red[k] = 0.0f;
                smem[k] = 0.0f;
                continue;
            }
            const uint16_t* src = grads + u.arena_pos + e;
            uint16_t gb[kSmallStepMaxRanks];
#pragma unroll
            for (int r = 0; r < kSmallStepMaxRanks; ++r)
                if (r < N) gb[r] = src[(int64_t)r * P_arena];
            const __nv_bfloat16 h = __float2bfloat16_rn(smem[k]);
            const uint16_t bits = *reinterpret_cast<const uint16_t*>(&h);
            ag[k] = bits;
            arena[u.arena_pos + e] = bits;
            float acc = bf16_bits_to_f32(gb[0]);
#pragma unroll
            for (int r = 1; r < kSmallStepMaxRanks; ++r)
                if (r < N) acc = __fadd_rn(acc, bf16_bits_to_f32(gb[r]));
            for (int r = kSmallStepMaxRanks; r < N; ++r)
                acc = __fadd_rn(acc, bf16_bits_to_f32(src[(int64_t)r * P_arena]));
            const float g = finish(acc, avg, fN);
            red[k] = g;
            smem[k] = g;
        }
    }
    __syncthreads();  // AdamW reads the reduced gradient of every rank
    // step 3: AdamW on the registers of step 1
#pragma unroll
    for (int j = 0; j < kStepPerThread; ++j) {
        const int64_t k = threadIdx.x + (int64_t)j * kStepThreads;
        if (k < count) {
            adamw1(pp[j], mm[j], vv[j], smem[k], sc);
            p[k] = pp[j];
            m[k] = mm[j];
            v[k] = vv[j];
        }
    }
}

}  // namespace

cudaError_t launch_small_step(const fsdp_group& g, float* master, float* m, float* v,
                              const uint16_t* grads, int op, uint16_t* ag, uint16_t* arena,
                              float* reduced, const AdamScalars& sc, const AdamScalars* sc_dev,
                              cudaStream_t st, const StepCounter& ctr) {
    const int64_t count = (int64_t)g.L * g.S;
    if (count == 0) return cudaSuccess;
    const int avg = (op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? 1 : 0;
    // one fp32 word per element: at most 32 KB, within the 48 KB of dynamic
    // shared memory a launch gets without opting in
    const size_t smem = (size_t)count * sizeof(float);
    k_small_step<<<1, kStepThreads, smem, st>>>(master, m, v, grads, g.P_arena, g.N, ag, arena,
                                                reduced, g.d_units, (int64_t)g.units.size(),
                                                count, avg, sc, sc_dev, ctr
                                                FSDPK_DBG_ARG(debug_bounds(g, kDbgSmallStep)));
    return cudaGetLastError();
}

}  // namespace fsdpk
