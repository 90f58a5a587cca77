/*
 * fsdpk.h -- C ABI of libfsdpk.so, the B200 (sm_100a) kernels of the FSDP2
 * per-parameter sharding step, with the N data-parallel ranks of one
 * parameter group emulated as N virtual ranks resident in one GPU's memory.
 *
 * Sources, by page title and section:
 *   [ML] "Sharded Training: FSDP2, DTensor, Tensor and Pipeline Parallelism":
 *        fully_shard paragraph (Shard(0): rank r keeps chunk r of
 *        torch.chunk(param, world, dim=0), padded internally when rows do not
 *        divide evenly; one fully_shard call = one parameter group = one unit
 *        of communication), Mixed precision paragraph (param_dtype bf16
 *        all-gather, reduce_dtype fp32 reduction), Other controls paragraph
 *        (set_force_sum_reduction_for_comms: SUM plus FSDP's own division),
 *        opening paragraph (2 + 2 + 12 bytes per parameter).
 *   [MS] "Introduction to PyTorch FSDP2 Backend Features": Working Principle
 *        (all-gather -> compute -> reduce-scatter -> sharded update) and
 *        Mixed Precision.
 *
 * Notation for a group of n parameters over N ranks (registration order i):
 *   d0_i = rows, cols_i = product of the remaining dims (1 for 1-D tensors)
 *   c_i  = ceil(d0_i / N)              rows of every rank's padded shard
 *   v_ir = clamp(d0_i - r*c_i, 0, c_i) real rows on rank r (the rest: pad)
 *   s_i  = c_i*cols_i; off_i = s_0 + ... + s_{i-1}; S = sum of s_i
 *   u_i  = unsharded ("arena") offset of parameter i: the previous
 *          parameter's end rounded up to a multiple of 8 elements (16 bytes);
 *          P_arena = last end rounded up to a multiple of 8.
 *   P    = sum of d0_i*cols_i (real elements of the group).
 *
 * Buffer layouts (element counts; all row-major, no strides):
 *   sharded fp32 state (master, m, v, reduced grad): [N][S], rank-major;
 *       rank r's shard of parameter i is rows [0, c_i) x cols_i at
 *       r*S + off_i; rows >= v_ir are padding and hold +0.
 *   all-gather buffer (bf16): [N][S], same layout as the sharded state.
 *   unsharded arena (bf16 params, fp32 full params): [P_arena], parameter i
 *       as a dense [d0_i][cols_i] block at u_i; gap elements are never
 *       read or written.
 *   per-rank full gradients (bf16): [N][P_arena], rank r's arena at
 *       r*P_arena.
 *   packed reduce-scatter input (fp32, optional): [N][N][S]; packed[r][j] is
 *       what rank r contributes to destination rank j.
 * bf16 values are passed as their uint16_t bit patterns.
 *
 * Ownership: the caller allocates and owns every data buffer and stream.  The
 * library owns only the plan (host tables and one device table, allocated in
 * fsdp_plan_group on the device current at that time, freed by
 * fsdp_destroy_group).  A plan is used on the device it was made on.
 *
 * Execution: every data call validates its arguments on the host, enqueues
 * kernels on `stream` and returns without synchronising.  Data pointers are
 * device pointers (or managed memory) and must be 16-byte aligned.  Buffers
 * of one call must not overlap unless stated.  Calls on the same group may run
 * concurrently on different streams only if their buffers are disjoint.
 *
 * Errors: every call returns an fsdp_status.  Invalid arguments are detected
 * before any launch and nothing is enqueued; FSDP_ECUDA reports a failed
 * launch (cudaGetLastError after the launch).  No kernel traps or waits.
 */
#ifndef FSDPK_H
#define FSDPK_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every entry point below is exported; the library hides everything else. */
#if defined(FSDPK_BUILDING_LIBRARY)
#define FSDP_API __attribute__((visibility("default")))
#else
#define FSDP_API
#endif

#define FSDP_MAX_NDIM 8
#define FSDP_MAX_WORLD 1024
#define FSDP_ABI_VERSION 1

/* One parameter's shape; dims must be >= 0, ndim in [0, FSDP_MAX_NDIM].
 * ndim == 0 (a scalar) is treated as shape [1]. */
typedef struct {
    int32_t ndim;
    int64_t shape[FSDP_MAX_NDIM];
} fsdp_param_desc;

/* Opaque plan of one parameter group (one fully_shard call). */
typedef struct fsdp_group* fsdp_group_t;

/* Same type as cudaStream_t; NULL is the legacy default stream. */
struct CUstream_st;
typedef struct CUstream_st* fsdp_stream_t;

typedef enum {
    FSDP_OK = 0,
    FSDP_EINVAL = -1, /* bad argument (null, size, count, op, hparams)     */
    FSDP_ENOMEM = -2, /* host or device allocation of the plan failed      */
    FSDP_ECUDA = -3,  /* a CUDA runtime call or kernel launch failed       */
    FSDP_EALIGN = -4, /* a data pointer is not 16-byte aligned             */
    FSDP_ESTATE = -5  /* call not valid now: plan used on a device other
                         than its own, a host-only plan given to a data
                         call, or (fsdp_rs_reduce_noalloc) a capturing
                         stream                                            */
} fsdp_status;

/* Reduce-scatter reduction ([ML] Other controls; The bug Adam hid). */
typedef enum {
    FSDP_SUM = 0,          /* ((g_0 + g_1) + ...) + g_{N-1}, binary32 RN   */
    FSDP_AVG = 1,          /* the SUM divided once by N (IEEE binary32 /)  */
    FSDP_SUM_THEN_DIV = 2  /* SUM, then FSDP's own division by N; the same
                              bits as FSDP_AVG                             */
} fsdp_reduce_op;

/* AdamW hyper-parameters (decoupled weight decay).  step is the 1-based
 * step count t used in the bias corrections 1 - beta^t. */
typedef struct {
    double lr;
    double beta1;
    double beta2;
    double eps;
    double weight_decay;
    int64_t step;
} fsdp_adamw_hparams;

/* One step's AdamW scalars in device memory (opaque, 32 bytes, 16-byte
 * aligned), written by fsdp_adamw_prepare and read by the *_dev entry
 * points, so that a captured CUDA graph advances the step count each time it
 * is replayed. */
typedef struct {
    float opaque[8];
} fsdp_adamw_dev_scalars;

/* ------------------------------------------------------------------------ */
/* Plan                                                                     */
/* ------------------------------------------------------------------------ */

/* Build the plan of one group: chunk rows, padded shard offsets, arena
 * offsets and the device work tables ([ML] fully_shard paragraph).
 * params: n_params descriptors (host memory, read only during the call).
 * n_params >= 0; world_size in [1, FSDP_MAX_WORLD].  On success *out owns a
 * new plan.  Errors: EINVAL (bad descriptor, sizes overflow int64),
 * ENOMEM, ECUDA (device table upload). */
FSDP_API int fsdp_plan_group(const fsdp_param_desc* params, int32_t n_params,
                    int32_t world_size, fsdp_group_t* out);

/* A plan built on the host only: the same layout and work tables as
 * fsdp_plan_group, with no CUDA call and no device memory, for inspecting and
 * checking a layout on a machine without a GPU.  Every data call refuses it
 * (FSDP_ESTATE, or FSDP_ECUDA where no device is present); destroy it with
 * fsdp_destroy_group. */
FSDP_API int fsdp_plan_group_host(const fsdp_param_desc* params, int32_t n_params,
                                  int32_t world_size, fsdp_group_t* out);

/* Checks the host copies of a plan's work tables against everything the data
 * calls assume: each unit inside [N][S] and inside its parameter's padded
 * shard, the units covering [N][S] exactly once, each real unit's arena
 * position recomputed from its shard position (the Shard(0) placement), pad
 * units on the pad rows, the pad intervals matching the pad units, and each
 * copy-in tile's interval range, the pack tables, and the flat path's
 * segment and vector-code tables recomputed from the units.  *violations
 * receives the number of failed checks (0 for every plan this library
 * builds).  Host only. */
FSDP_API int fsdp_group_check(fsdp_group_t group, int64_t* violations);

/* Which work tables the data calls of a plan use -- an inspection of the
 * group plan of "Sharded Training: FSDP2, DTensor, Tensor and Pipeline
 * Parallelism", fully_shard paragraph (one group per call, rows chunked and
 * padded per rank); the pages describe no such choice.  A group of many small
 * parameters (at least 2048 short and pad runs, both index spaces below 2^30
 * elements) takes the flat path in the bf16 copy-out, the fused
 * reduce-scatter and the bf16 fused update: fixed tiles of the index space,
 * one code per 8-element vector, instead of one work unit per (rank,
 * parameter) run -- the same results, bit for bit.  The copy-out takes it
 * only when runs shorter than 1024 elements hold at least a tenth of the real
 * elements (with mostly long runs the per-run copy-out is faster).  *flat
 * receives bit 0 set for a plan whose reduce-scatter and update are flat,
 * bit 1 for a flat copy-out, else 0; *mixed_shard and *mixed_arena the
 * vectors of the [N][S] and of the arena index space that hold more than one
 * run (or a run and padding, or the ragged end), which go element by element
 * (0 where that side is not flat).  Host only; any output pointer may be
 * NULL.
 * Errors: FSDP_EINVAL (NULL group). */
FSDP_API int fsdp_group_flat(fsdp_group_t group, int32_t* flat, int64_t* mixed_shard,
                             int64_t* mixed_arena);

/* S (per-rank padded shard elements), P (real elements), P_arena of a plan:
 * the sizes of one rank's padded shard of the group and of the unsharded
 * group ("Sharded Training: FSDP2, DTensor, Tensor and Pipeline
 * Parallelism", fully_shard paragraph: each rank keeps chunk r of
 * torch.chunk along dim 0, padded when the rows do not divide).  Host only;
 * any output pointer may be NULL.  Errors: FSDP_EINVAL (NULL group). */
FSDP_API int fsdp_group_sizes(fsdp_group_t group, int64_t* S, int64_t* P,
                     int64_t* P_arena);

/* Per-parameter tables, each an int64 array of n_params entries supplied by
 * the caller (any may be NULL): off_i (where parameter i's padded shard
 * starts inside a rank's [S] slot), u_i (its start in the unsharded arena)
 * and c_i (the torch.chunk chunk rows, ceil(d0_i / N)) -- the per-parameter
 * placement of the same fully_shard paragraph.  Host only.
 * Errors: FSDP_EINVAL (NULL group). */
FSDP_API int fsdp_group_param_offsets(fsdp_group_t group, int64_t* shard_off,
                             int64_t* arena_off, int64_t* chunk_rows);

/* Free a plan (NULL is ignored): its host tables and its device table.  The
 * plan is one fully_shard group's pre-computed layout, which FSDP2 keeps for
 * the life of the module ("PyTorch FSDP2 Guide: Distributed LLM Training with
 * DTensor", The Architecture, section 2: buffers are planned once and
 * reused), so this is called once, at tear-down.  Work already enqueued that
 * uses the plan must have completed. */
FSDP_API void fsdp_destroy_group(fsdp_group_t group);

/* ------------------------------------------------------------------------ */
/* Data path (asynchronous on `stream`)                                     */
/* ------------------------------------------------------------------------ */

/* Shard(0) placement: fp32 full parameters in arena layout [P_arena] ->
 * padded fp32 master [N][S] (pad rows written as +0).  This is fully_shard's
 * initial sharding ([ML] fully_shard paragraph). */
FSDP_API int fsdp_shard_params(fsdp_group_t group, const float* full_arena,
                      float* master, fsdp_stream_t stream);

/* Stage 1, all-gather copy-in: ag[r][k] = bf16_rn(master[r][k]) for real
 * elements and +0 for pad elements ([ML] Mixed precision: bf16 copies are
 * all-gathered; [MS] Mixed Precision).  master: fp32 [N][S] (read);
 * ag: bf16 [N][S] (written). */
FSDP_API int fsdp_copy_in(fsdp_group_t group, const float* master, uint16_t* ag,
                 fsdp_stream_t stream);

/* Stage 2, all-gather copy-out: the rank-major buffer is split into the
 * unsharded parameters with the padding stripped ([MS] Working Principle,
 * All-Gather state): arena[u_i + row*cols_i + col] =
 * ag[r*S + off_i + (row - r*c_i)*cols_i + col] with r = row / c_i.
 * ag: bf16 [N][S] (read); arena: bf16 [P_arena] (written, gaps untouched). */
FSDP_API int fsdp_copy_out(fsdp_group_t group, const uint16_t* ag, uint16_t* arena,
                  fsdp_stream_t stream);

/* Stages 3 + 4, reduce-scatter: each rank's bf16 full gradients are cast to
 * fp32 (reduce_dtype), packed per destination rank and reduced over the N
 * ranks in rank order ([ML] Mixed precision, Other controls).
 * grads: bf16 [N][P_arena] (read).  reduced: fp32 [N][S] (written; pads +0).
 * op: an fsdp_reduce_op.  packed_or_null: NULL runs the fused path (no
 * packed buffer is materialised); otherwise fp32 [N][N][S] receives the packed
 * reduce-scatter inputs and the reduction reads them back (staged path; for
 * FSDP_SUM_THEN_DIV the division is a separate pass).  Both paths give the
 * same bits. */
FSDP_API int fsdp_rs_reduce(fsdp_group_t group, const uint16_t* grads, int32_t op,
                   float* packed_or_null, float* reduced,
                   fsdp_stream_t stream);

/* Stage 5, sharded AdamW on all N*S elements (decoupled weight decay,
 * PyTorch's documented AdamW; [ML] Fence 4 and opening paragraph: 12 bytes
 * of fp32 state per parameter):
 *   p <- p*(1 - lr*wd);  m <- b1*m + (1-b1)*g;  v <- b2*v + (1-b2)*g*g
 *   p <- p - (lr/(1-b1^t)) * m / (sqrt(v)/sqrt(1-b2^t) + eps)
 * master, m, v: fp32 [N][S] updated in place; grad: fp32 [N][S] (read).
 * A zero pad stays +0.  hparams: host pointer; step >= 1, lr >= 0,
 * 0 <= beta < 1, eps > 0.  Computed in binary32. */
FSDP_API int fsdp_adamw_step(fsdp_group_t group, float* master, float* m, float* v,
                    const float* grad, const fsdp_adamw_hparams* hparams,
                    fsdp_stream_t stream);

/* Stages 3 + 4 + 5 fused, followed by the next step's stage 1: the
 * reduce-scatter of fsdp_rs_reduce (fused path), the AdamW update of
 * fsdp_adamw_step on the reduced gradient, and the copy-in of
 * fsdp_copy_in on the updated master, in one pass over [N][S].  It follows the
 * lifecycle of [MS] Working Principle (reduce-scatter, then the sharded
 * update, then the next all-gather): the reduced gradient stays in registers
 * and the updated fp32 master is cast while it is still in registers.
 * Results are the same bits as running fsdp_rs_reduce, fsdp_adamw_step and
 * fsdp_copy_in in turn.
 *   grads: bf16 [N][P_arena] (read); op: an fsdp_reduce_op;
 *   master, m, v: fp32 [N][S] (updated in place); hparams as for
 *   fsdp_adamw_step;
 *   ag_next_or_null: bf16 [N][S] receiving bf16_rn(updated master), +0 in
 *   pad rows (the next all-gather's input), or NULL;
 *   reduced_or_null: fp32 [N][S] receiving the reduced gradient, or NULL.
 * Algorithmic bytes: 2N per real element + 24 (+2 with ag, +4 with reduced)
 * per padded element.  Errors as for fsdp_rs_reduce and fsdp_adamw_step. */
FSDP_API int fsdp_rs_adamw_step(fsdp_group_t group, const uint16_t* grads, int32_t op,
                       float* master, float* m, float* v,
                       const fsdp_adamw_hparams* hparams,
                       uint16_t* ag_next_or_null, float* reduced_or_null,
                       fsdp_stream_t stream);

/* Groups with N*S at most this many elements run fsdp_group_step as one
 * single-CTA launch. */
#define FSDP_SMALL_STEP_ELEMS 8192

/* The whole step of one group, stages 1-5 in the order of [MS] Working
 * Principle: fsdp_copy_in of the pre-update master into ag, fsdp_copy_out of
 * ag into arena, the fused fsdp_rs_reduce of grads into reduced, and
 * fsdp_adamw_step with reduced.  Same bits as those four calls in turn.
 * Groups with N*S <= FSDP_SMALL_STEP_ELEMS run as ONE launch of a single CTA
 * (for them the launches, not the bytes, are the cost; a block barrier
 * separates dependent stages); larger groups as the four stage kernels on
 * `stream`.
 *   master, m, v: fp32 [N][S] (updated); grads: bf16 [N][P_arena] (read);
 *   op: an fsdp_reduce_op; hparams as for fsdp_adamw_step; ag: bf16 [N][S]
 *   (written); arena: bf16 [P_arena] (written, gaps untouched); reduced:
 *   fp32 [N][S] (written).  All 16-byte aligned.
 * fsdp_group_step_dev takes the AdamW scalars from device memory (written
 * by fsdp_adamw_prepare), for a step captured in a CUDA graph.
 * Errors as for the four stage calls. */
FSDP_API int fsdp_group_step(fsdp_group_t group, float* master, float* m, float* v,
                             const uint16_t* grads, int32_t op,
                             const fsdp_adamw_hparams* hparams, uint16_t* ag,
                             uint16_t* arena, float* reduced, fsdp_stream_t stream);

FSDP_API int fsdp_group_step_dev(fsdp_group_t group, float* master, float* m, float* v,
                                 const uint16_t* grads, int32_t op,
                                 const fsdp_adamw_dev_scalars* scalars_dev, uint16_t* ag,
                                 uint16_t* arena, float* reduced, fsdp_stream_t stream);

/* The whole step of one group as ONE call that a CUDA graph can replay as
 * successive training steps ("Introduction to PyTorch FSDP2 Backend
 * Features", Working Principle: all-gather, reduce-scatter, update, in that
 * order): fsdp_adamw_prepare and fsdp_group_step_dev in one.  It advances
 * the device step counter *step_dev, computes that step's AdamW scalars on
 * the device (left in *scalars_dev) and runs the step.  A group with
 * N*S <= FSDP_SMALL_STEP_ELEMS is one launch in all (its single CTA advances
 * the counter and computes the scalars itself, while its first loads are in
 * flight); a larger group is the prepare kernel and the four stage kernels.
 * Same bits as fsdp_adamw_prepare followed by fsdp_group_step_dev.
 *   hparams: lr, betas, eps, weight_decay as for fsdp_adamw_step (step is
 *   ignored); step_dev: device int64, 8-byte aligned, 0 before the first
 *   step; scalars_dev: device memory, 16-byte aligned; the other arguments
 *   as for fsdp_group_step.
 * Errors as for fsdp_adamw_prepare and fsdp_group_step. */
FSDP_API int fsdp_group_step_graph(fsdp_group_t group, float* master, float* m, float* v,
                                   const uint16_t* grads, int32_t op,
                                   const fsdp_adamw_hparams* hparams, int64_t* step_dev,
                                   fsdp_adamw_dev_scalars* scalars_dev, uint16_t* ag,
                                   uint16_t* arena, float* reduced, fsdp_stream_t stream);

/* Gradient accumulation without sync ([ML] Other controls:
 * set_requires_gradient_sync(False) accumulates the unsharded gradients and
 * skips the reduce-scatter).  Each rank's unsharded gradient is accumulated in
 * reduce_dtype fp32, a left fold over microbatches:
 *   first != 0: acc[k] = fp32(grads[k]);  first == 0: acc[k] += fp32(grads[k])
 * over every element of [N][P_arena] (gap elements included; they are never
 * read by the reduce-scatter).  grads: bf16 [N][P_arena] (read); acc: fp32
 * [N][P_arena] (updated; not read when first != 0).  Algorithmic bytes per
 * element: 6 (first) or 10. */
FSDP_API int fsdp_grad_accumulate(fsdp_group_t group, const uint16_t* grads, float* acc,
                         int32_t first, fsdp_stream_t stream);

/* The reduce-scatter of the last microbatch when gradients were accumulated:
 * for each rank, x_r = acc_r (+ fp32(grads_r) when grads_or_null is not
 * NULL, the last microbatch's own gradient), then the packing and the
 * rank-ordered fold of fsdp_rs_reduce on the fp32 x_r.  Equal to
 * fsdp_grad_accumulate(grads) followed by a reduce-scatter of acc, without
 * writing acc back.  acc: fp32 [N][P_arena] (read); reduced: fp32 [N][S]
 * (written, pads +0).  Algorithmic bytes: 6N (4N without grads) per real
 * element + 4 per padded element. */
FSDP_API int fsdp_rs_reduce_accumulated(fsdp_group_t group, const uint16_t* grads_or_null,
                               const float* acc, int32_t op, float* reduced,
                               fsdp_stream_t stream);

/* The all-gather copy-in and copy-out with param_dtype fp32 (no
 * MixedPrecisionPolicy: [ML] Mixed precision), a test mode: nothing is cast,
 * so fsdp_copy_out_f32(fsdp_copy_in_f32(shard(x))) == x bit for bit.
 *   fsdp_copy_in_f32: master fp32 [N][S] (read) -> ag32 fp32 [N][S] (written,
 *   +0 in pad rows).  fsdp_copy_out_f32: ag32 -> arena32 fp32 [P_arena]
 *   (written on real elements, gaps untouched).  16-byte aligned pointers.
 * Algorithmic bytes: 8 per padded element (copy-in), 8 per real element
 * (copy-out). */
FSDP_API int fsdp_copy_in_f32(fsdp_group_t group, const float* master, float* ag32,
                              fsdp_stream_t stream);
FSDP_API int fsdp_copy_out_f32(fsdp_group_t group, const float* ag32, float* arena32,
                               fsdp_stream_t stream);

/* FP8 all-gather copy-in ("PyTorch FSDP2 Guide: Distributed LLM Training
 * with DTensor", Deep Dive, "2. Native FP8 Training with Float8Tensor":
 * parameters in FP8 E4M3, the all-gather moves raw FP8 bytes).  The page
 * leaves the scaling open; this library uses per-parameter tensorwise
 * dynamic scaling:
 *   amax_i  = max |master| over parameter i, all ranks (NaN ignored)
 *   scale_i = 448 / max(amax_i, 1e-12)                       (binary32)
 *   ag8[r][k] = e4m3_rn(clamp(master[r][k] * scale_i, -448, 448)),
 * 0x00 in pad rows; E4M3 is the "fn" encoding (no infinities, largest
 * finite 448).  A consumer recovers x ~ e4m3_value(q) / scale_i.
 * master: fp32 [N][S] (read); ag8: uint8 [N][S] (written); scales: fp32
 * [n_params] (written; 4-byte aligned).  Algorithmic bytes: 4 (amax pass) +
 * 4 + 1 per padded element. */
FSDP_API int fsdp_copy_in_fp8(fsdp_group_t group, const float* master, uint8_t* ag8,
                     float* scales, fsdp_stream_t stream);

/* FP8 copy-in with given scales (no amax pass): ag8 as for fsdp_copy_in_fp8
 * with scale_i = scales[i] supplied by the caller, e.g. the previous step's
 * scales in delayed scaling.  master: fp32 [N][S] (read); scales: fp32
 * [n_params] (read; 4-byte aligned); ag8: uint8 [N][S] (written, 0x00 in
 * pad rows).  Algorithmic bytes: 4 + 1 per padded element. */
FSDP_API int fsdp_copy_in_fp8_scaled(fsdp_group_t group, const float* master,
                                     const float* scales, uint8_t* ag8,
                                     fsdp_stream_t stream);

/* fsdp_rs_adamw_step with an FP8 next all-gather input (delayed scaling):
 * the reduce-scatter and AdamW update of fsdp_rs_adamw_step, then, while the
 * updated master is in registers,
 *   ag8_next[r][k] = e4m3_rn(clamp(master[r][k] * scales_prev[i], -448, 448))
 * (0x00 in pad rows) and the next scales from the updated master,
 *   scales_next[i] = 448 / max(max |master| over parameter i, 1e-12),
 * the scale rule of fsdp_copy_in_fp8.  The scales lag one step behind the
 * master they quantise: the amax is known only after the update has passed
 * over the whole parameter, and reading the master again to apply it would
 * cost the 4 bytes per element the fusion saves.  The result equals
 * fsdp_rs_reduce + fsdp_adamw_step + fsdp_copy_in_fp8_scaled(scales_prev),
 * and scales_next equals the scales fsdp_copy_in_fp8 computes from the
 * updated master.
 *   grads, op, master, m, v, hparams, reduced_or_null: as for
 *   fsdp_rs_adamw_step;  scales_prev: fp32 [n_params] (read);
 *   ag8_next: uint8 [N][S] (written); scales_next: fp32 [n_params] (written;
 *   a different buffer from scales_prev).  Both scale buffers 4-byte aligned.
 * Algorithmic bytes: 2N per real element + 25 (+4 with reduced) per padded
 * element.  Three launches on `stream`: a memset of scales_next, the fused
 * kernel and a per-parameter division. */
FSDP_API int fsdp_rs_adamw_step_fp8(fsdp_group_t group, const uint16_t* grads, int32_t op,
                                    float* master, float* m, float* v,
                                    const fsdp_adamw_hparams* hparams,
                                    const float* scales_prev, uint8_t* ag8_next,
                                    float* scales_next, float* reduced_or_null,
                                    fsdp_stream_t stream);

/* FP8 copy-out: the byte-for-byte counterpart of fsdp_copy_out.
 * ag8: uint8 [N][S] (read); arena8: uint8 [P_arena] (written, gaps
 * untouched).  Algorithmic bytes: 1 read + 1 written per real element. */
FSDP_API int fsdp_copy_out_fp8(fsdp_group_t group, const uint8_t* ag8, uint8_t* arena8,
                      fsdp_stream_t stream);

/* Graph-replayable AdamW.  fsdp_adamw_step and fsdp_rs_adamw_step take the
 * step count t from the host, so a captured CUDA graph would replay the same
 * t; these entry points read it from device memory instead.
 * fsdp_adamw_prepare enqueues one thread that sets *step_dev += 1 and writes
 * the scalars of that step (decay 1 - lr*wd, lr / (1 - beta1^t),
 * 1 / sqrt(1 - beta2^t), ...; computed in binary64 on the device, as the host
 * path computes them) to *scalars_dev.  hparams->step is ignored; the other
 * fields are validated as for fsdp_adamw_step.  step_dev: device int64,
 * 8-byte aligned, set to 0 by the caller before the first step;
 * scalars_dev: device memory, 16-byte aligned.  One prepare per step serves
 * every group that shares the hyper-parameters.
 * fsdp_adamw_step_dev and fsdp_rs_adamw_step_dev are fsdp_adamw_step and
 * fsdp_rs_adamw_step with the scalars read from scalars_dev (written by a
 * prepare earlier on the same stream). */
FSDP_API int fsdp_adamw_prepare(const fsdp_adamw_hparams* hparams, int64_t* step_dev,
                                fsdp_adamw_dev_scalars* scalars_dev, fsdp_stream_t stream);

FSDP_API int fsdp_adamw_step_dev(fsdp_group_t group, float* master, float* m, float* v,
                                 const float* grad, const fsdp_adamw_dev_scalars* scalars_dev,
                                 fsdp_stream_t stream);

FSDP_API int fsdp_rs_adamw_step_dev(fsdp_group_t group, const uint16_t* grads, int32_t op,
                                    float* master, float* m, float* v,
                                    const fsdp_adamw_dev_scalars* scalars_dev,
                                    uint16_t* ag_next_or_null, float* reduced_or_null,
                                    fsdp_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Reduce-scatter without any allocation                                    */
/* ------------------------------------------------------------------------ */

/* Largest work table fsdp_rs_reduce_noalloc accepts: one table entry per run
 * of at most 8192 elements of a (rank, parameter) shard segment, so this
 * covers groups of up to about 1.07e9 padded elements (N*S) when the
 * segments are large. */
#define FSDP_NOALLOC_MAX_UNITS 131072

/* The fused reduce-scatter of fsdp_rs_reduce (packed_or_null == NULL), for
 * callers that cannot allocate device memory: a custom allocator or memory
 * pool that owns every byte of the device, code running where cudaMalloc is
 * forbidden (inside another library's critical section, a process whose
 * memory budget is fixed up front).  There is no plan object: the group is
 * described by params / n_params / world_size exactly as for
 * fsdp_plan_group, and the work table the kernel needs is written into a
 * fixed array in the library's own device memory (FSDP_NOALLOC_MAX_UNITS
 * entries of 24 bytes, 3 MiB on every GPU that loads the library, held until
 * the process exits).  The call itself makes no cudaMalloc, cudaFree or
 * other allocating call.  (The pages describe no counterpart of this entry
 * point.)
 *   grads: bf16 [N][P_arena] (read); reduced: fp32 [N][S] (written, pads
 *   +0); op: an fsdp_reduce_op; results are bit-identical to fsdp_rs_reduce.
 *   P_arena and S follow the layout rules at the top of this file; the
 *   library cannot see the sizes of the caller's buffers, so they must hold
 *   at least N*P_arena and N*S elements.
 * Set-up: the CUDA runtime loads the library's device code, and with it the
 * 3 MiB array, on the first call on each device (lazy module loading).  Make
 * that first call at set-up time, before the device's memory is handed to a
 * pool.  Every call looks the array's address up on the current device.
 * Ordering: the table is built on the host and copied into the array with
 * cudaMemcpyAsync on `stream` from pageable host memory, so each call waits
 * for the work already queued on `stream` before it returns (the copy from
 * pageable memory synchronises with the stream), and the driver stages the
 * copy through its own buffers.  That copy reads a host array that the next
 * call overwrites, so while `stream` is being captured into a CUDA graph the
 * call returns FSDP_ESTATE and enqueues nothing.
 * Every call shares the one array and leaves its last table there: calls on
 * the same device that overlap on the GPU (different streams without
 * ordering between them) race; serialise them on one stream.  Host threads
 * are serialised inside the call.
 * Errors: FSDP_EINVAL for the same argument errors as fsdp_plan_group and
 * fsdp_rs_reduce, and for a group that needs more than
 * FSDP_NOALLOC_MAX_UNITS table entries (nothing is enqueued then);
 * FSDP_EALIGN; FSDP_ESTATE (stream capture, see above); FSDP_ECUDA. */
FSDP_API int fsdp_rs_reduce_noalloc(const fsdp_param_desc* params, int32_t n_params,
                           int32_t world_size, const uint16_t* grads, int32_t op,
                           float* reduced, fsdp_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Several devices: the exchange steps as pulls over peer memory            */
/* ------------------------------------------------------------------------ */

/* With D devices (one process per GPU), device d holds the L = N / D virtual
 * ranks [d*L, (d+1)*L) of a group: their master, m, v shards and reduced
 * gradients, fp32 [L][S]; their all-gather slot, bf16 [L][S] (the copy-in
 * output, rank-major like the [N][S] buffer it is a slice of); and their
 * unsharded gradients, bf16 [L][P_arena].  The group's two exchange steps
 * ("Introduction to PyTorch FSDP2 Backend Features", Working Principle: the
 * all-gather before the parameters are used, the reduce-scatter after the
 * backward pass) become pulls inside the stage kernels, over NVLink when a
 * source lives on another GPU:
 *   copy-out  reads each rank's rows straight from that rank's slot row;
 *   reduce    reads each source rank's gradient arena and folds the N ranks
 *             in rank order 0..N-1, the same bits as on one device.
 * The caller maps the other devices' buffers into its address space
 * (fsdp_ipc_*) and passes one pointer per rank.  Ordering across devices is
 * the caller's: a slot row must be complete before any copy-out reads it and
 * must not be rewritten (by a copy-in or a fused update) while one still
 * reads it; a gradient arena must be complete before any reduction reads it.
 * Pulls are plain loads; no kernel waits on another device. */

#define FSDP_PEER_MAX_RANKS 64

typedef struct fsdp_peer* fsdp_peer_t;

/* The plan of device `device_index` of `n_devices` for `group`: N must be a
 * multiple of n_devices and N <= FSDP_PEER_MAX_RANKS.  `group` must outlive
 * the peer plan (its copy-out table is shared).  n_devices == 1 is allowed
 * (every rank local).  Allocates the local work tables and the two pointer
 * tables on the current device, which must be the group's.
 * Errors: FSDP_EINVAL, FSDP_ESTATE (other device), FSDP_ENOMEM, FSDP_ECUDA. */
FSDP_API int fsdp_peer_plan(fsdp_group_t group, int32_t n_devices, int32_t device_index,
                            fsdp_peer_t* out);

/* Sizes of the local buffers: L ranks, first rank r0. */
FSDP_API int fsdp_peer_local_ranks(fsdp_peer_t peer, int32_t* L, int32_t* r0);

/* Where every rank's data lives.  ag_rank_ptrs: host array of N device
 * pointers, entry r = the first element of rank r's bf16 slot row (S
 * elements), 2-byte aligned; grad_rank_ptrs: host array of N device
 * pointers, entry r = rank r's bf16 gradient arena (P_arena elements),
 * 16-byte aligned.  Either array may be NULL to keep the previous table.
 * Pointers may be this device's or mapped from peers; they are copied to the
 * device synchronously (the slot rows as one source pointer per copy-out
 * work unit, resolved here, so the copy-out kernel does no rank lookup).  Errors: FSDP_EINVAL (NULL entry where S or
 * P_arena > 0), FSDP_EALIGN, FSDP_ECUDA. */
FSDP_API int fsdp_peer_set_sources(fsdp_peer_t peer, const uint16_t* const* ag_rank_ptrs,
                                   const uint16_t* const* grad_rank_ptrs);

/* Release the peer plan's tables (not the group, not any data buffer). */
FSDP_API void fsdp_destroy_peer_plan(fsdp_peer_t peer);

/* Copy-in of the local ranks: master fp32 [L][S] -> ag_slot bf16 [L][S], as
 * fsdp_copy_in for these ranks (pads +0). */
FSDP_API int fsdp_peer_copy_in(fsdp_peer_t peer, const float* master, uint16_t* ag_slot,
                               fsdp_stream_t stream);

/* Copy-out of all N ranks into this device's unsharded arena (bf16
 * [P_arena], gaps untouched), pulling rank r's rows from ag_rank_ptrs[r].
 * Same bits as fsdp_copy_out of the gathered [N][S] buffer.  Needs the
 * all-gather table (FSDP_ESTATE otherwise). */
FSDP_API int fsdp_peer_copy_out(fsdp_peer_t peer, uint16_t* arena, fsdp_stream_t stream);

/* The fused reduce-scatter for the local destination ranks: reduced fp32
 * [L][S] (pads +0) from the N gradient arenas of grad_rank_ptrs, in rank
 * order; same bits as the local rows of fsdp_rs_reduce.  Needs the gradient
 * table (FSDP_ESTATE otherwise). */
FSDP_API int fsdp_peer_rs_reduce(fsdp_peer_t peer, int32_t op, float* reduced,
                                 fsdp_stream_t stream);

/* AdamW on the local shards (fp32 [L][S]), as fsdp_adamw_step. */
FSDP_API int fsdp_peer_adamw_step(fsdp_peer_t peer, float* master, float* m, float* v,
                                  const float* grad, const fsdp_adamw_hparams* hparams,
                                  fsdp_stream_t stream);

/* fsdp_rs_adamw_step for the local ranks: the pull reduce-scatter, AdamW on
 * master/m/v fp32 [L][S], and optionally the next copy-in into ag_next_or_null
 * (bf16 [L][S], normally this device's slot) and the reduced gradient into
 * reduced_or_null (fp32 [L][S]).  Same bits as the local rows of
 * fsdp_rs_adamw_step. */
FSDP_API int fsdp_peer_rs_adamw_step(fsdp_peer_t peer, int32_t op, float* master, float* m,
                                     float* v, const fsdp_adamw_hparams* hparams,
                                     uint16_t* ag_next_or_null, float* reduced_or_null,
                                     fsdp_stream_t stream);

/* The FP8 all-gather over several devices (delayed scaling, as
 * fsdp_rs_adamw_step_fp8): each device's slot holds E4M3 bytes [L][S], so the
 * copy-out pulls half the bytes.  The per-parameter amax spans every rank, so
 * each device folds the maximum of its own rows into a partial amax array
 * (uint32 [n_params], the bits of a non-negative float) and the scales are
 * the maximum over the devices' partial arrays: one more exchange, of
 * 4 * n_params bytes per device.
 * fsdp_peer_set_fp8_sources: ag8_rank_ptrs, host array of N device pointers
 * (entry r = rank r's E4M3 slot row, S bytes); amax_device_ptrs, host array
 * of n_devices device pointers (device d's partial amax array, 4-byte
 * aligned).  Resolved and copied to the device synchronously.
 * fsdp_peer_copy_in_fp8_scaled: fsdp_copy_in_fp8_scaled for the local ranks
 * (master fp32 [L][S] -> ag8_slot uint8 [L][S], scales fp32 [n_params]).
 * fsdp_peer_copy_out_fp8: fsdp_copy_out_fp8 of all N ranks into arena8
 * (uint8 [P_arena]), pulling each rank's bytes from its slot row.
 * fsdp_peer_rs_adamw_step_fp8: fsdp_rs_adamw_step_fp8 for the local ranks,
 * except that the amax of the updated local rows goes to amax_local (zeroed
 * first) instead of the next scales; ag8_next is normally the device's own
 * slot.  fsdp_peer_fp8_scales: scales_next[i] = 448 / max(max over devices
 * of partial amax i, 1e-12), reading every device's array (after a barrier
 * that follows every device's fused update).  The scales, slots and arena
 * then equal those of fsdp_rs_adamw_step_fp8 and fsdp_copy_out_fp8 on one
 * device.  Errors as for the single-device calls; FSDP_ESTATE before the
 * tables are set. */
FSDP_API int fsdp_peer_set_fp8_sources(fsdp_peer_t peer, const uint8_t* const* ag8_rank_ptrs,
                                       const uint32_t* const* amax_device_ptrs);
FSDP_API int fsdp_peer_copy_in_fp8_scaled(fsdp_peer_t peer, const float* master,
                                          const float* scales, uint8_t* ag8_slot,
                                          fsdp_stream_t stream);
FSDP_API int fsdp_peer_copy_out_fp8(fsdp_peer_t peer, uint8_t* arena8, fsdp_stream_t stream);
FSDP_API int fsdp_peer_rs_adamw_step_fp8(fsdp_peer_t peer, int32_t op, float* master, float* m,
                                         float* v, const fsdp_adamw_hparams* hparams,
                                         const float* scales_prev, uint8_t* ag8_next,
                                         uint32_t* amax_local, float* reduced_or_null,
                                         fsdp_stream_t stream);
FSDP_API int fsdp_peer_fp8_scales(fsdp_peer_t peer, float* scales_next, fsdp_stream_t stream);

/* Device memory other processes can map (CUDA IPC).  fsdp_ipc_alloc
 * allocates `bytes` (> 0) on the current device with cudaMalloc and writes
 * the handle another process passes to fsdp_ipc_open; free it with
 * fsdp_ipc_free once no process has it open.  fsdp_ipc_open maps a handle
 * from another process (any device of this node that can access the owner's
 * memory) at *ptr, with peer access enabled lazily; fsdp_ipc_close unmaps
 * it.  A handle cannot be opened in the process that allocated it.
 * Errors: FSDP_EINVAL (null arguments, bytes <= 0), FSDP_ENOMEM,
 * FSDP_ECUDA. */
typedef struct {
    uint8_t bytes[64];
} fsdp_ipc_handle;

FSDP_API int fsdp_ipc_alloc(int64_t bytes, void** ptr, fsdp_ipc_handle* handle);
FSDP_API int fsdp_ipc_free(void* ptr);
FSDP_API int fsdp_ipc_open(const fsdp_ipc_handle* handle, void** ptr);
FSDP_API int fsdp_ipc_close(void* ptr);

/* ------------------------------------------------------------------------ */
/* Misc                                                                     */
/* ------------------------------------------------------------------------ */

/* Static description of a status code (never NULL; unknown codes get a
 * generic text).  The pages define no error model; the codes are this
 * library's, so that nothing throws across the C ABI. */
FSDP_API const char* fsdp_status_string(int status);

/* The cudaError_t of the most recent FSDP_ECUDA on this thread (0 if none). */
FSDP_API int fsdp_last_cuda_error(void);

/* Debug build.  libfsdpk_debug.so is the same library compiled with
 * -DFSDPK_DEBUG: every kernel that indexes memory through a plan's work
 * tables checks each work unit (and each copy-in tile's pad-interval range)
 * against the extents of the buffers the launch was given -- the [L][S]
 * buffers, one unsharded arena, the pad-interval or parameter table -- before
 * touching memory through it.  A unit that would reach outside is skipped and
 * counted; nothing traps and nothing waits.  The pages describe no
 * counterpart (their lab guards runs only with a wall-clock limit).
 * fsdp_debug_build: 1 in the debug library, 0 otherwise.
 * fsdp_debug_set_error_words: `words` is a caller-owned device buffer of 4
 * uint32 (4-byte aligned; NULL to stop recording) on the device of the
 * launches that follow: words[0] counts violations (one per warp that sees
 * one), words[1..3] hold the first one's kernel id, unit or tile index and
 * block index.  The caller zeroes it and reads it.  `shrink` (>= 0, tests
 * only) narrows every launch's extents by that many elements, so that valid
 * tables trip the checks without any access leaving the real buffers.  The
 * setting is process-wide and read at each launch.
 * Errors: FSDP_ESTATE in a release library; FSDP_EINVAL (shrink < 0);
 * FSDP_EALIGN. */
FSDP_API int fsdp_debug_build(void);
FSDP_API int fsdp_debug_set_error_words(uint32_t* words, int64_t shrink);

/* FSDP_ABI_VERSION of the loaded library. */
FSDP_API int fsdp_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FSDPK_H */
