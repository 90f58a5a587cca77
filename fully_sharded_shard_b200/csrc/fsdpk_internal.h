// fsdpk_internal.h -- types shared by the plan builder, the kernels and the
// C-ABI entry points of libfsdpk.so.  Not part of the public interface.
#pragma once

#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "fsdpk.h"

namespace fsdpk {

// Elements per work unit of the segment kernels (copy-out, reduce-scatter,
// pack, shard).  Large enough that a unit's head/tail peeling is noise,
// small enough that the largest parameter splits into thousands of units.
constexpr int64_t kUnitElems = 8192;

// Elements per tile of the flat copy-in kernel (256 threads x 8 x 4).
constexpr int64_t kCopyInTile = 8192;

// The copy-outs give each real unit of at least kShortRun elements a CTA of
// its own; shorter units (small parameters, the last piece of a split run)
// are packed, up to kPackUnits units and kPackElems elements per CTA, one
// warp per unit.
constexpr int64_t kShortRun = 1024;
constexpr int64_t kPackUnits = 64;
constexpr int64_t kPackElems = 16384;

// Flat path of a group of many small parameters (at least kFlatMinUnits
// short and pad units): the fused reduce-scatter, the fused update and the
// copy-out run over fixed tiles of the flat index space instead of over
// units, reading one code per 16-byte vector of 8 bf16 elements:
//   even, not kFlatPad: all 8 elements are real rows of one run, and
//                       element k's other-side position is k + code / 2
//   kFlatPad:           all 8 elements are pad rows (shard side) or arena
//                       gaps (arena side)
//   odd, 2 m + 1:       mixed (several runs, a run and pads or gaps, or the
//                       partial last vector): entry m of the mixed list, whose
//                       vector index is mixq[m] and whose elements' codes
//                       (2 * offset, or kFlatPad; kFlatPad past the end) are
//                       mixc[8 m .. 8 m + 7].  A second launch takes the
//                       mixed vectors, a thread per element.
// Codes are int32, so both index spaces stay below kFlatMaxElems.
constexpr int64_t kFlatMinUnits = 2048;
// The copy-out reads 2 B and writes 2 B per element, so a code's 0.5 B per
// element weighs more there: it takes the flat path only when runs shorter
// than kShortRun hold at least 1 / kFlatCopyOutShare of the real elements
// (with mostly long runs the per-unit copy-out is the faster one).
constexpr int64_t kFlatCopyOutShare = 10;
constexpr int64_t kFlatMaxElems = (int64_t{1} << 30) - 64;
constexpr int32_t kFlatPad = INT32_MIN;

// A maximal range of a flat index space with one code (2 * offset to the
// other side, or kFlatPad), running to the next segment's start; the last
// segment of a table is a sentinel at the end of the space.  Host side only:
// the codes and the mixed lists are built from these segments.
struct FlatSeg {
    int32_t start;
    int32_t code;
};

// One contiguous run of a (rank j, parameter i) shard segment.
//   shard_pos: first element in the rank-major [N][S] index space
//   arena_pos: first element of the matching rows in an unsharded arena
//              (real runs only)
//   len:       elements in the run
//   is_pad:    1 for a run of pad rows (written as +0), 0 for real rows
struct Unit {
    int64_t shard_pos;
    int64_t arena_pos;
    int32_t len;
    int32_t is_pad;
};
static_assert(sizeof(Unit) == 24, "Unit layout");

// A half-open range [lo, hi) of pad elements in the [N][S] index space.
struct Interval {
    int64_t lo;
    int64_t hi;
};

// For each copy-in tile, the half-open index range of the pad intervals that
// intersect it.
struct TileRange {
    int32_t begin;
    int32_t end;
};

// Debug build (-DFSDPK_DEBUG): the extents a table-driven kernel checks every
// work unit (or tile) against before touching memory through it.  A unit that
// would reach outside is skipped and counted in the caller's error words
// (fsdp_debug_set_error_words); nothing traps and nothing waits.
struct DebugBounds {
    int64_t ns;       // elements of the [L][S] buffers that shard positions index
    int64_t arena;    // elements of one unsharded arena that arena positions index
    int64_t n_aux;    // entries of the side table the kernel indexes (pad
                      // intervals, or parameters for the FP8 kernels)
    uint32_t* words;  // [count, kernel id, unit or tile index, block], or null
    int32_t kernel;   // DebugKernel of the launch
};

// Kernel ids recorded with the first violation.
enum DebugKernel : int32_t {
    kDbgCopyIn = 1, kDbgCopyOut, kDbgCopyOutTab, kDbgShard, kDbgReduce, kDbgReduceTab,
    kDbgRsAdamw, kDbgRsAdamwTab, kDbgReduceAcc, kDbgFp8Amax, kDbgFp8CopyIn, kDbgFp8CopyOut,
    kDbgFp8CopyOutTab, kDbgSmallStep, kDbgCopyInF32, kDbgCopyOutF32, kDbgReduceFlat,
    kDbgRsAdamwFlat, kDbgCopyOutFlat
};

}  // namespace fsdpk

// The opaque plan behind fsdp_group_t.
struct fsdp_group {
    int device = -1;
    int sm_count = 0;
    int32_t N = 0;  // virtual ranks of the group (sources of every reduction)
    int32_t L = 0;  // ranks whose shards this plan's [L][S] buffers hold: N, or
                    // N / D for the local view of a device's D-way peer plan
    int32_t n = 0;
    std::vector<int64_t> d0, cols, c, s, off, u;
    int64_t S = 0, P = 0, P_arena = 0;
    int64_t pad_elems = 0;  // N*S - P

    // host copies (kept for inspection and tests of the plan); shard
    // positions index the [L][S] buffers
    std::vector<fsdpk::Unit> units;  // real units first, then pad units; the real
                                     // units of kShortRun elements or more first
    std::vector<int32_t> unit_param;  // parameter index of every unit
    int64_t n_real_units = 0;
    int64_t n_long_units = 0;        // real units [0, n_long_units) are long
    std::vector<int32_t> packs;      // pack p = units [packs[p], packs[p + 1]),
                                     // packs[0] = n_long_units, back = n_real_units
    std::vector<int32_t> rpacks;     // the reduce-scatter's packs: the short real
                                     // units and every pad unit, [n_long_units, units)
    std::vector<fsdpk::Interval> intervals;
    std::vector<fsdpk::TileRange> tile_ranges;  // empty when no padding
    int64_t n_tiles = 0;                        // copy-in tiles over L*S
    // flat path (empty unless flat): codes of the shard-side vectors of
    // [L][S] and of the arena-side vectors of [P_arena], with their segments
    bool flat = false;           // reduce-scatter and update
    bool flat_copy_out = false;  // the copy-out too (amap, amixq, amixc)
    std::vector<int32_t> smap, amap;    // one code per vector
    std::vector<int32_t> smixq, amixq;  // the mixed vectors
    std::vector<int32_t> smixc, amixc;  // their elements' codes, 8 per vector
    std::vector<fsdpk::FlatSeg> ssegs, asegs;

    // one device allocation holding the tables
    void* dev_mem = nullptr;
    const fsdpk::Unit* d_units = nullptr;
    const fsdpk::Interval* d_intervals = nullptr;
    const fsdpk::TileRange* d_tile_ranges = nullptr;
    const int32_t* d_unit_param = nullptr;
    const int32_t* d_packs = nullptr;
    const int32_t* d_rpacks = nullptr;
    const int32_t* d_smap = nullptr;
    const int32_t* d_smixq = nullptr;
    const int32_t* d_smixc = nullptr;
    const int32_t* d_amap = nullptr;
    const int32_t* d_amixq = nullptr;
    const int32_t* d_amixc = nullptr;
};

// The opaque peer plan behind fsdp_peer_t: device `index` of `n_devices` holds the
// virtual ranks [r0, r0 + L) of `parent`'s group.
struct fsdp_peer {
    const fsdp_group* parent = nullptr;  // copy-out units of all N ranks; not owned
    fsdp_group local;                    // tables of the local ranks, local coordinates
    int32_t n_devices = 0;
    int32_t index = 0;
    int64_t r0 = 0;
    // one device allocation: N gradient arena pointers, one bf16 source
    // pointer per copy-out unit of the parent, one FP8 source pointer per
    // copy-out unit, then n_devices amax-array pointers (set by
    // fsdp_peer_set_sources and fsdp_peer_set_fp8_sources)
    void* dev_tab = nullptr;
    bool have_ag = false;
    bool have_grads = false;
    bool have_fp8 = false;
};

namespace fsdpk {

// Plan helpers (fsdpk_api.cu): the work tables of ranks [r0, r1) in local
// coordinates, their upload, their release, and the recording of a CUDA
// error for fsdp_last_cuda_error.  Return FSDP status codes.
int build_rank_tables(fsdp_group* g, int64_t r0, int64_t r1);
int upload_tables(fsdp_group* g);
void free_tables(fsdp_group* g);
int record_cuda_error(cudaError_t e);
// FSDP_OK when the current device is g's, FSDP_ESTATE (or FSDP_ECUDA) otherwise.
int check_plan_device(const fsdp_group* g);

// The bounds of a launch over g's tables (debug build; the words and the
// test-only shrink come from fsdp_debug_set_error_words).
DebugBounds debug_bounds(const fsdp_group& g, int32_t kernel, int64_t n_aux = 0);
DebugBounds debug_bounds_raw(int64_t ns, int64_t arena, int32_t kernel, int64_t n_aux = 0);

// Scalars of one AdamW step, precomputed on the host in binary64.
struct AdamScalars {
    float decay;         // 1 - lr*wd
    float beta1, omb1;   // b1, 1 - b1
    float beta2, omb2;   // b2, 1 - b2
    float step_size;     // lr / (1 - b1^t)
    float inv_bc2_sqrt;  // 1 / sqrt(1 - b2^t)
    float eps;
};
static_assert(sizeof(AdamScalars) == 32, "AdamScalars is the 32-byte fsdp_adamw_dev_scalars");

// A device step counter that a kernel advances itself (a graph-replayed
// step), with the hyper-parameters of the scalars it then computes and where
// to leave them (out may be null).  step == nullptr: no counter.
struct StepCounter {
    int64_t* step = nullptr;
    AdamScalars* out = nullptr;
    double lr = 0, beta1 = 0, beta2 = 0, eps = 0, wd = 0;
};

// Validate AdamW hyper-parameters and compute one step's scalars (binary64).
bool host_adam_scalars(const fsdp_adamw_hparams* hp, AdamScalars* sc);

// Kernel launchers (fsdpk_gather.cu, fsdpk_reduce.cu, fsdpk_update.cu).  They enqueue work and return the
// cudaError_t of the launch.
cudaError_t launch_copy_in(const fsdp_group& g, const float* master, uint16_t* ag,
                           cudaStream_t st);
cudaError_t launch_copy_out(const fsdp_group& g, const uint16_t* ag, uint16_t* arena,
                            cudaStream_t st);
cudaError_t launch_rs_fused(const fsdp_group& g, const uint16_t* grads, int op,
                            float* reduced, cudaStream_t st);
cudaError_t launch_rs_pack(const fsdp_group& g, const uint16_t* grads, float* packed,
                           cudaStream_t st);
cudaError_t launch_rs_reduce_packed(const fsdp_group& g, const float* packed, int op,
                                    float* reduced, cudaStream_t st);
cudaError_t launch_div_inplace(const fsdp_group& g, float* reduced, cudaStream_t st);
cudaError_t launch_adamw(const fsdp_group& g, float* master, float* m, float* v,
                         const float* grad, const AdamScalars& sc, cudaStream_t st,
                         const AdamScalars* sc_dev = nullptr);
// Advance *step on the device and write that step's scalars to *out.
cudaError_t launch_adamw_prepare(double lr, double beta1, double beta2, double eps, double wd,
                                 int64_t* step, AdamScalars* out, cudaStream_t st);
cudaError_t launch_shard(const fsdp_group& g, const float* full, float* master,
                         cudaStream_t st);
// The fused reduce-scatter over a caller-supplied unit table (device memory)
// instead of a plan's own table.
cudaError_t launch_rs_fused_units(int sm_count, int N, int64_t P_arena, const Unit* units,
                                  int64_t n_units, const uint16_t* grads, int op, float* reduced,
                                  cudaStream_t st, int64_t NS);

// The exchange steps over pointer tables in device memory: the copy-out
// pulling each of the parent's real units from unit_src[unit] (inside the
// slot row of the unit's rank), and the reductions folding rank r's gradient
// arena at grad_tab[r] (N pointers).  `parent` supplies the copy-out units,
// `local` the units of the local destination ranks.
cudaError_t launch_copy_out_tab(const fsdp_group& parent, const uint16_t* const* unit_src,
                                uint16_t* arena, cudaStream_t st);
cudaError_t launch_rs_fused_tab(const fsdp_group& local, const uint16_t* const* grad_tab, int op,
                                float* reduced, cudaStream_t st);
cudaError_t launch_rs_adamw_tab(const fsdp_group& local, const uint16_t* const* grad_tab, int op,
                                float* master, float* m, float* v, const AdamScalars& sc,
                                uint16_t* ag_next, float* reduced, cudaStream_t st);
// The FP8 forms: the byte copy-out pulling each unit from unit_src8[unit],
// the fused update writing the local E4M3 slot and the local partial amax
// bits, and the scales from the devices' partial amax arrays (amax_tab: a
// device array of D pointers).
cudaError_t launch_copy_out_fp8_tab(const fsdp_group& parent, const uint8_t* const* unit_src8,
                                    uint8_t* arena8, cudaStream_t st);
cudaError_t launch_rs_adamw_tab_fp8(const fsdp_group& local, const uint16_t* const* grad_tab,
                                    int op, float* master, float* m, float* v,
                                    const AdamScalars& sc, const float* scales_prev,
                                    uint8_t* ag8_next, unsigned* amax_bits, float* reduced,
                                    cudaStream_t st);
cudaError_t launch_fp8_scales_from_parts(const unsigned* const* amax_tab, int D, float* scales,
                                         int n, cudaStream_t st);

// The whole step of a small group (copy-in, copy-out, fused reduce-scatter,
// AdamW) in one single-CTA launch (fsdpk_step.cu).
cudaError_t launch_small_step(const fsdp_group& g, float* master, float* m, float* v,
                              const uint16_t* grads, int op, uint16_t* ag, uint16_t* arena,
                              float* reduced, const AdamScalars& sc, const AdamScalars* sc_dev,
                              cudaStream_t st, const StepCounter& ctr = StepCounter{});

// Fused reduce-scatter + AdamW (+ optional next-step copy-in into ag_next and
// optional reduced-gradient output).
cudaError_t launch_rs_adamw(const fsdp_group& g, const uint16_t* grads, int op, float* master,
                            float* m, float* v, const AdamScalars& sc, uint16_t* ag_next,
                            float* reduced, cudaStream_t st, const AdamScalars* sc_dev = nullptr);

// Gradient accumulation without sync over [N][P_arena] in fp32, and the
// reduce-scatter of the accumulated arenas (+ the last microbatch's bf16
// gradients when grads is not null).
cudaError_t launch_accumulate(const fsdp_group& g, const uint16_t* grads, float* acc, int first,
                              cudaStream_t st);
cudaError_t launch_rs_reduce_acc(const fsdp_group& g, const uint16_t* grads, const float* acc,
                                 int op, float* reduced, cudaStream_t st);

// FP8 (E4M3) all-gather: per-parameter scales from the master's amax, the
// quantising copy-in and the byte copy-out.
cudaError_t launch_copy_in_fp8(const fsdp_group& g, const float* master, uint8_t* ag8,
                               float* scales, cudaStream_t st);
cudaError_t launch_copy_out_fp8(const fsdp_group& g, const uint8_t* ag8, uint8_t* arena8,
                                cudaStream_t st);

// FP8 with given scales: scales from amax in place, and the copy-in with
// scales supplied by the caller (no amax pass).
cudaError_t launch_fp8_scales_from_amax(const fsdp_group& g, float* scales, cudaStream_t st);
cudaError_t launch_copy_in_fp8_scaled(const fsdp_group& g, const float* master, uint8_t* ag8,
                                      const float* scales, cudaStream_t st);
// The fused update writing the next all-gather input in FP8 with delayed
// scales and folding max |updated master| per parameter into amax_bits.
cudaError_t launch_rs_adamw_fp8(const fsdp_group& g, const uint16_t* grads, int op, float* master,
                                float* m, float* v, const AdamScalars& sc, const float* scales_prev,
                                uint8_t* ag8_next, unsigned* amax_bits, float* reduced,
                                cudaStream_t st, const AdamScalars* sc_dev = nullptr);

}  // namespace fsdpk
