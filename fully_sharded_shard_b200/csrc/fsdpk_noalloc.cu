// fsdpk_noalloc.cu -- fsdp_rs_reduce_noalloc: the fused reduce-scatter for
// callers that cannot allocate device memory (see include/fsdpk.h).
//
// The work table that fsdp_plan_group would upload into a cudaMalloc'd
// buffer lives here in a fixed array in the library's own device memory.
// Host code never uses the array's name as a pointer (in host code it is
// only a stand-in for the device symbol); every call looks the device
// address up with cudaGetSymbolAddress on the current device and passes
// that address on, so a device reset or another context never leaves a
// stale address behind.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "fsdpk.h"
#include "fsdpk_internal.h"

namespace {

constexpr int64_t kMaxUnits = FSDP_NOALLOC_MAX_UNITS;

// The shared work table: FSDP_NOALLOC_MAX_UNITS x 24 bytes on every device
// that loads the library.  Only the first n_units entries of the current
// call are read, and the call writes all of them first, so nothing in it
// has to start at zero.
static __device__ __align__(256) fsdpk::Unit g_noalloc_units[kMaxUnits];

// Host staging copy of the table (static storage, not allocated per call).
// One mutex serialises host threads.  The copy to the device reads this
// array when the call enqueues it, so a call is refused while its stream is
// being captured: a captured copy would read whatever table a later call
// left here each time the graph is replayed.
std::mutex g_mu;
fsdpk::Unit g_host_units[kMaxUnits];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool mul_ok(int64_t a, int64_t b, int64_t* out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / a) return false;
    *out = a * b;
    return true;
}

bool add_ok(int64_t a, int64_t b, int64_t* out) {
    if (b > INT64_MAX - a) return false;
    *out = a + b;
    return true;
}

// Rows and columns of one descriptor (ndim 0 is a scalar, shape [1]).
bool rows_cols(const fsdp_param_desc& d, int64_t* d0, int64_t* cols) {
    if (d.ndim < 0 || d.ndim > FSDP_MAX_NDIM) return false;
    *d0 = 1;
    *cols = 1;
    for (int k = 0; k < d.ndim; ++k) {
        if (d.shape[k] < 0) return false;
        if (k == 0) *d0 = d.shape[0];
        else if (!mul_ok(*cols, d.shape[k], cols)) return false;
    }
    return true;
}

// Append the runs of [shard_pos, shard_pos + len) as table entries of at
// most kUnitElems elements; false when the table is full.
bool push(int64_t* n, int64_t shard_pos, int64_t arena_pos, int64_t len, int32_t is_pad) {
    for (int64_t done = 0; done < len; done += fsdpk::kUnitElems) {
        if (*n >= kMaxUnits) return false;
        const int64_t l = std::min<int64_t>(fsdpk::kUnitElems, len - done);
        g_host_units[*n] = fsdpk::Unit{shard_pos + done, is_pad ? 0 : arena_pos + done,
                                       (int32_t)l, is_pad};
        ++*n;
    }
    return true;
}

}  // namespace

extern "C" int fsdp_rs_reduce_noalloc(const fsdp_param_desc* params, int32_t n_params,
                                      int32_t world_size, const uint16_t* grads, int32_t op,
                                      float* reduced, fsdp_stream_t stream) {
    if (n_params < 0 || (n_params > 0 && params == nullptr)) return FSDP_EINVAL;
    if (world_size < 1 || world_size > FSDP_MAX_WORLD) return FSDP_EINVAL;
    if (op != FSDP_SUM && op != FSDP_AVG && op != FSDP_SUM_THEN_DIV) return FSDP_EINVAL;
    if (!aligned16(grads) || !aligned16(reduced)) return FSDP_EALIGN;
    const int64_t N = world_size;

    // pass 1: S, P and the arena size (same layout rules as fsdp_plan_group)
    int64_t S = 0, P = 0, A = 0;
    for (int32_t i = 0; i < n_params; ++i) {
        int64_t d0, cols, s, numel, u;
        if (!rows_cols(params[i], &d0, &cols)) return FSDP_EINVAL;
        const int64_t c = d0 == 0 ? 0 : (d0 + N - 1) / N;
        if (!mul_ok(c, cols, &s) || !mul_ok(d0, cols, &numel)) return FSDP_EINVAL;
        if (!add_ok(S, s, &S) || !add_ok(P, numel, &P) || !add_ok(A, 7, &u)) return FSDP_EINVAL;
        u = u / 8 * 8;
        if (!add_ok(u, numel, &A)) return FSDP_EINVAL;
    }
    int64_t A8, NS, NA, tmp;
    if (!add_ok(A, 7, &A8)) return FSDP_EINVAL;
    const int64_t P_arena = A8 / 8 * 8;
    if (!mul_ok(N, S, &NS) || !mul_ok(N, P_arena, &NA) || !mul_ok(NS, 4, &tmp) ||
        !mul_ok(NA, 2, &tmp))
        return FSDP_EINVAL;
    if (NS > 0 && reduced == nullptr) return FSDP_EINVAL;
    if (P > 0 && grads == nullptr) return FSDP_EINVAL;

    cudaStream_t st = (cudaStream_t)stream;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    const cudaError_t qe = cudaStreamIsCapturing(st, &cap);
    if (qe == cudaErrorStreamCaptureImplicit) {  // the legacy stream while another captures
        (void)cudaGetLastError();
        return FSDP_ESTATE;
    }
    if (qe != cudaSuccess) return FSDP_ECUDA;
    if (cap != cudaStreamCaptureStatusNone) return FSDP_ESTATE;

    std::lock_guard<std::mutex> lock(g_mu);

    // the array's address on the current device (the first call on a device
    // loads the library's device code and this array there)
    void* dev_units = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&dev_units, g_noalloc_units);
    if (e != cudaSuccess || dev_units == nullptr) return FSDP_ECUDA;

    // pass 2: the table -- real runs for every (rank j, parameter i), then pads
    int64_t n_units = 0;
    for (int pass = 0; pass < 2; ++pass) {
        for (int64_t j = 0; j < N; ++j) {
            int64_t off = 0, a = 0;
            for (int32_t i = 0; i < n_params; ++i) {
                int64_t d0, cols;
                rows_cols(params[i], &d0, &cols);
                const int64_t c = d0 == 0 ? 0 : (d0 + N - 1) / N;
                const int64_t u = (a + 7) / 8 * 8;
                const int64_t v = std::clamp<int64_t>(d0 - j * c, 0, c);
                bool ok;
                if (pass == 0)
                    ok = push(&n_units, j * S + off, u + j * c * cols, v * cols, 0);
                else
                    ok = push(&n_units, j * S + off + v * cols, 0, (c - v) * cols, 1);
                if (!ok) return FSDP_EINVAL;  // more than FSDP_NOALLOC_MAX_UNITS entries
                off += c * cols;
                a = u + d0 * cols;
            }
        }
    }
    if (n_units == 0) return FSDP_OK;

    e = cudaMemcpyAsync(dev_units, g_host_units, (size_t)n_units * sizeof(fsdpk::Unit),
                        cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return FSDP_ECUDA;
    // the grid covers the units once and does not depend on the SM count
    e = fsdpk::launch_rs_fused_units(0, world_size, P_arena,
                                     static_cast<const fsdpk::Unit*>(dev_units), n_units, grads,
                                     op, reduced, st, NS);
    return e == cudaSuccess ? FSDP_OK : FSDP_ECUDA;
}
