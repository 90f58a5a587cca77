// fsdpk_peer.cu -- host side of the multi-device exchange: the peer plan of
// one device (the work tables of its local virtual ranks; one gradient-arena
// pointer per rank; one source pointer per copy-out work unit into the bf16
// and the FP8 slot rows, resolved here; one partial-amax pointer per device),
// its entry points, and the CUDA IPC helpers that map other processes'
// buffers.
//
// The exchange steps of "Introduction to PyTorch FSDP2 Backend Features",
// Working Principle (all-gather before use, reduce-scatter after backward)
// run as pulls inside the copy-out and reduction kernels: each rank's data
// is read where it lives, over NVLink when that is another GPU, and the
// reduction keeps the rank order 0..N-1 of the single-device path.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "fsdpk.h"
#include "fsdpk_internal.h"

namespace {

int cuda_status(cudaError_t e) {
    return e == cudaSuccess ? FSDP_OK : fsdpk::record_cuda_error(e);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

const uint16_t* const* grad_table(const fsdp_peer* p) {
    return static_cast<const uint16_t* const*>(p->dev_tab);
}

const uint16_t* const* unit_src_table(const fsdp_peer* p) {
    return static_cast<const uint16_t* const*>(p->dev_tab) + p->parent->N;
}

void* const* table_base(const fsdp_peer* p) { return static_cast<void* const*>(p->dev_tab); }

const uint8_t* const* unit_src8_table(const fsdp_peer* p) {
    return reinterpret_cast<const uint8_t* const*>(table_base(p) + p->parent->N +
                                                   p->parent->n_real_units);
}

const unsigned* const* amax_table(const fsdp_peer* p) {
    return reinterpret_cast<const unsigned* const*>(table_base(p) + p->parent->N +
                                                    2 * p->parent->n_real_units);
}

int check_op(int32_t op) {
    return (op == FSDP_SUM || op == FSDP_AVG || op == FSDP_SUM_THEN_DIV) ? FSDP_OK : FSDP_EINVAL;
}

}  // namespace

extern "C" {

int fsdp_peer_plan(fsdp_group_t g, int32_t n_devices, int32_t device_index, fsdp_peer_t* out) {
    if (out == nullptr) return FSDP_EINVAL;
    *out = nullptr;
    if (g == nullptr || n_devices < 1 || device_index < 0 || device_index >= n_devices)
        return FSDP_EINVAL;
    if (g->L != g->N || g->N % n_devices != 0 || g->N > FSDP_PEER_MAX_RANKS) return FSDP_EINVAL;
    int st = fsdpk::check_plan_device(g);
    if (st != FSDP_OK) return st;
    fsdp_peer* p = new (std::nothrow) fsdp_peer();
    if (p == nullptr) return FSDP_ENOMEM;
    p->parent = g;
    p->n_devices = n_devices;
    p->index = device_index;
    const int32_t L = g->N / n_devices;
    p->r0 = (int64_t)device_index * L;
    fsdp_group& l = p->local;
    try {
        l.N = g->N;
        l.L = L;
        l.n = g->n;
        l.d0 = g->d0;
        l.cols = g->cols;
        l.c = g->c;
        l.s = g->s;
        l.off = g->off;
        l.u = g->u;
        l.S = g->S;
        l.P = g->P;
        l.P_arena = g->P_arena;
        l.pad_elems = g->pad_elems;
    } catch (...) {
        delete p;
        return FSDP_ENOMEM;
    }
    st = fsdpk::build_rank_tables(&l, p->r0, p->r0 + L);
    if (st == FSDP_OK) st = fsdpk::upload_tables(&l);
    if (st == FSDP_OK) {
        cudaError_t e = cudaMalloc(&p->dev_tab, ((size_t)g->N + 2 * (size_t)g->n_real_units +
                                                 (size_t)n_devices) *
                                                    sizeof(void*));
        if (e != cudaSuccess) {
            cudaGetLastError();
            p->dev_tab = nullptr;
            st = e == cudaErrorMemoryAllocation ? FSDP_ENOMEM : cuda_status(e);
        }
    }
    if (st != FSDP_OK) {
        fsdpk::free_tables(&l);
        delete p;
        return st;
    }
    *out = p;
    return FSDP_OK;
}

int fsdp_peer_local_ranks(fsdp_peer_t p, int32_t* L, int32_t* r0) {
    if (p == nullptr) return FSDP_EINVAL;
    if (L) *L = p->local.L;
    if (r0) *r0 = (int32_t)p->r0;
    return FSDP_OK;
}

int fsdp_peer_set_sources(fsdp_peer_t p, const uint16_t* const* ag_rank_ptrs,
                          const uint16_t* const* grad_rank_ptrs) {
    if (p == nullptr) return FSDP_EINVAL;
    const int32_t N = p->parent->N;
    for (int32_t r = 0; ag_rank_ptrs != nullptr && r < N; ++r) {
        if (p->parent->S > 0 && ag_rank_ptrs[r] == nullptr) return FSDP_EINVAL;
        if (reinterpret_cast<uintptr_t>(ag_rank_ptrs[r]) & 1u) return FSDP_EALIGN;
    }
    for (int32_t r = 0; grad_rank_ptrs != nullptr && r < N; ++r) {
        if (p->parent->P_arena > 0 && grad_rank_ptrs[r] == nullptr) return FSDP_EINVAL;
        if (!aligned16(grad_rank_ptrs[r])) return FSDP_EALIGN;
    }
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    const size_t bytes = (size_t)N * sizeof(void*);
    cudaError_t e = cudaSuccess;
    if (ag_rank_ptrs != nullptr && p->parent->n_real_units > 0) {
        // each copy-out unit's source: its rank's slot row + its offset in it
        std::vector<const uint16_t*> src;
        try {
            src.resize((size_t)p->parent->n_real_units);
        } catch (...) {
            return FSDP_ENOMEM;
        }
        const int64_t S = p->parent->S;
        for (int64_t ui = 0; ui < p->parent->n_real_units; ++ui) {
            const int64_t pos = p->parent->units[(size_t)ui].shard_pos;
            const int64_t r = pos / S;  // a unit never crosses a rank's row
            src[(size_t)ui] = ag_rank_ptrs[r] + (pos - r * S);
        }
        e = cudaMemcpy(static_cast<char*>(p->dev_tab) + bytes, src.data(),
                       src.size() * sizeof(void*), cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess && grad_rank_ptrs != nullptr)
        e = cudaMemcpy(p->dev_tab, grad_rank_ptrs, bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_status(e);
    if (ag_rank_ptrs != nullptr) p->have_ag = true;
    if (grad_rank_ptrs != nullptr) p->have_grads = true;
    return FSDP_OK;
}

int fsdp_peer_set_fp8_sources(fsdp_peer_t p, const uint8_t* const* ag8_rank_ptrs,
                              const uint32_t* const* amax_device_ptrs) {
    if (p == nullptr || ag8_rank_ptrs == nullptr || amax_device_ptrs == nullptr)
        return FSDP_EINVAL;
    const int32_t N = p->parent->N;
    for (int32_t r = 0; r < N; ++r)
        if (p->parent->S > 0 && ag8_rank_ptrs[r] == nullptr) return FSDP_EINVAL;
    for (int32_t d = 0; d < p->n_devices; ++d) {
        if (p->parent->n > 0 && amax_device_ptrs[d] == nullptr) return FSDP_EINVAL;
        if (reinterpret_cast<uintptr_t>(amax_device_ptrs[d]) & 3u) return FSDP_EALIGN;
    }
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    std::vector<const void*> tab;
    try {
        tab.resize((size_t)p->parent->n_real_units + (size_t)p->n_devices);
    } catch (...) {
        return FSDP_ENOMEM;
    }
    const int64_t S = p->parent->S;
    for (int64_t ui = 0; ui < p->parent->n_real_units; ++ui) {
        const int64_t pos = p->parent->units[(size_t)ui].shard_pos;
        const int64_t r = pos / S;  // a unit never crosses a rank's row
        tab[(size_t)ui] = ag8_rank_ptrs[r] + (pos - r * S);
    }
    for (int32_t d = 0; d < p->n_devices; ++d)
        tab[(size_t)p->parent->n_real_units + (size_t)d] = amax_device_ptrs[d];
    void* dst = const_cast<void**>(table_base(p) + N + p->parent->n_real_units);
    cudaError_t e = cudaMemcpy(dst, tab.data(), tab.size() * sizeof(void*), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_status(e);
    p->have_fp8 = true;
    return FSDP_OK;
}

int fsdp_peer_copy_in_fp8_scaled(fsdp_peer_t p, const float* master, const float* scales,
                                 uint8_t* ag8_slot, fsdp_stream_t stream) {
    if (p == nullptr) return FSDP_EINVAL;
    const int64_t LS = (int64_t)p->local.L * p->local.S;
    if (LS > 0 && (master == nullptr || ag8_slot == nullptr)) return FSDP_EINVAL;
    if (p->local.n > 0 && scales == nullptr) return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(ag8_slot) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return FSDP_EALIGN;
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    return cuda_status(fsdpk::launch_copy_in_fp8_scaled(p->local, master, ag8_slot, scales,
                                                        (cudaStream_t)stream));
}

int fsdp_peer_copy_out_fp8(fsdp_peer_t p, uint8_t* arena8, fsdp_stream_t stream) {
    if (p == nullptr) return FSDP_EINVAL;
    if (p->parent->P > 0 && arena8 == nullptr) return FSDP_EINVAL;
    if (!aligned16(arena8)) return FSDP_EALIGN;
    if (!p->have_fp8) return FSDP_ESTATE;
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    return cuda_status(fsdpk::launch_copy_out_fp8_tab(*p->parent, unit_src8_table(p), arena8,
                                                      (cudaStream_t)stream));
}

int fsdp_peer_rs_adamw_step_fp8(fsdp_peer_t p, int32_t op, float* master, float* m, float* v,
                                const fsdp_adamw_hparams* hp, const float* scales_prev,
                                uint8_t* ag8_next, uint32_t* amax_local, float* reduced,
                                fsdp_stream_t stream) {
    if (p == nullptr || hp == nullptr || check_op(op) != FSDP_OK) return FSDP_EINVAL;
    const int64_t LS = (int64_t)p->local.L * p->local.S;
    if (LS > 0 && (master == nullptr || m == nullptr || v == nullptr || ag8_next == nullptr))
        return FSDP_EINVAL;
    if (p->local.n > 0 && (scales_prev == nullptr || amax_local == nullptr)) return FSDP_EINVAL;
    fsdpk::AdamScalars sc;
    if (!fsdpk::host_adam_scalars(hp, &sc)) return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(ag8_next) ||
        !aligned16(reduced) || (reinterpret_cast<uintptr_t>(scales_prev) & 3u) ||
        (reinterpret_cast<uintptr_t>(amax_local) & 3u))
        return FSDP_EALIGN;
    if (!p->have_grads) return FSDP_ESTATE;
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    if (p->local.n > 0) e = cudaMemsetAsync(amax_local, 0, sizeof(uint32_t) * (size_t)p->local.n, s);
    if (e == cudaSuccess)
        e = fsdpk::launch_rs_adamw_tab_fp8(p->local, grad_table(p), op, master, m, v, sc,
                                           scales_prev, ag8_next, amax_local, reduced, s);
    return cuda_status(e);
}

int fsdp_peer_fp8_scales(fsdp_peer_t p, float* scales_next, fsdp_stream_t stream) {
    if (p == nullptr) return FSDP_EINVAL;
    if (p->local.n > 0 && scales_next == nullptr) return FSDP_EINVAL;
    if (reinterpret_cast<uintptr_t>(scales_next) & 3u) return FSDP_EALIGN;
    if (!p->have_fp8) return FSDP_ESTATE;
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    return cuda_status(fsdpk::launch_fp8_scales_from_parts(amax_table(p), p->n_devices,
                                                           scales_next, p->local.n,
                                                           (cudaStream_t)stream));
}

void fsdp_destroy_peer_plan(fsdp_peer_t p) {
    if (p == nullptr) return;
    int prev = -1;
    bool switched = false;
    if (cudaGetDevice(&prev) == cudaSuccess && prev != p->local.device)
        switched = cudaSetDevice(p->local.device) == cudaSuccess;
    if (p->dev_tab) cudaFree(p->dev_tab);
    if (switched) cudaSetDevice(prev);
    fsdpk::free_tables(&p->local);
    delete p;
}

int fsdp_peer_copy_in(fsdp_peer_t p, const float* master, uint16_t* ag_slot,
                      fsdp_stream_t stream) {
    if (p == nullptr) return FSDP_EINVAL;
    const int64_t LS = (int64_t)p->local.L * p->local.S;
    if (LS > 0 && (master == nullptr || ag_slot == nullptr)) return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(ag_slot)) return FSDP_EALIGN;
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    return cuda_status(fsdpk::launch_copy_in(p->local, master, ag_slot, (cudaStream_t)stream));
}

int fsdp_peer_copy_out(fsdp_peer_t p, uint16_t* arena, fsdp_stream_t stream) {
    if (p == nullptr) return FSDP_EINVAL;
    if (p->parent->P > 0 && arena == nullptr) return FSDP_EINVAL;
    if (!aligned16(arena)) return FSDP_EALIGN;
    if (!p->have_ag) return FSDP_ESTATE;
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    return cuda_status(
        fsdpk::launch_copy_out_tab(*p->parent, unit_src_table(p), arena, (cudaStream_t)stream));
}

int fsdp_peer_rs_reduce(fsdp_peer_t p, int32_t op, float* reduced, fsdp_stream_t stream) {
    if (p == nullptr || check_op(op) != FSDP_OK) return FSDP_EINVAL;
    if ((int64_t)p->local.L * p->local.S > 0 && reduced == nullptr) return FSDP_EINVAL;
    if (!aligned16(reduced)) return FSDP_EALIGN;
    if (!p->have_grads) return FSDP_ESTATE;
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    return cuda_status(
        fsdpk::launch_rs_fused_tab(p->local, grad_table(p), op, reduced, (cudaStream_t)stream));
}

int fsdp_peer_adamw_step(fsdp_peer_t p, float* master, float* m, float* v, const float* grad,
                         const fsdp_adamw_hparams* hp, fsdp_stream_t stream) {
    if (p == nullptr || hp == nullptr) return FSDP_EINVAL;
    const int64_t LS = (int64_t)p->local.L * p->local.S;
    if (LS > 0 && (master == nullptr || m == nullptr || v == nullptr || grad == nullptr))
        return FSDP_EINVAL;
    fsdpk::AdamScalars sc;
    if (!fsdpk::host_adam_scalars(hp, &sc)) return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(grad))
        return FSDP_EALIGN;
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    return cuda_status(
        fsdpk::launch_adamw(p->local, master, m, v, grad, sc, (cudaStream_t)stream));
}

int fsdp_peer_rs_adamw_step(fsdp_peer_t p, int32_t op, float* master, float* m, float* v,
                            const fsdp_adamw_hparams* hp, uint16_t* ag_next, float* reduced,
                            fsdp_stream_t stream) {
    if (p == nullptr || hp == nullptr || check_op(op) != FSDP_OK) return FSDP_EINVAL;
    const int64_t LS = (int64_t)p->local.L * p->local.S;
    if (LS > 0 && (master == nullptr || m == nullptr || v == nullptr)) return FSDP_EINVAL;
    fsdpk::AdamScalars sc;
    if (!fsdpk::host_adam_scalars(hp, &sc)) return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(ag_next) ||
        !aligned16(reduced))
        return FSDP_EALIGN;
    if (!p->have_grads) return FSDP_ESTATE;
    int st = fsdpk::check_plan_device(&p->local);
    if (st != FSDP_OK) return st;
    return cuda_status(fsdpk::launch_rs_adamw_tab(p->local, grad_table(p), op, master, m, v, sc,
                                                  ag_next, reduced, (cudaStream_t)stream));
}

int fsdp_ipc_alloc(int64_t bytes, void** ptr, fsdp_ipc_handle* handle) {
    if (ptr == nullptr || handle == nullptr || bytes <= 0) return FSDP_EINVAL;
    *ptr = nullptr;
    static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(fsdp_ipc_handle), "IPC handle size");
    void* p = nullptr;
    cudaError_t e = cudaMalloc(&p, (size_t)bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e == cudaErrorMemoryAllocation ? FSDP_ENOMEM : cuda_status(e);
    }
    cudaIpcMemHandle_t h;
    e = cudaIpcGetMemHandle(&h, p);
    if (e != cudaSuccess) {
        cudaFree(p);
        return cuda_status(e);
    }
    std::memcpy(handle->bytes, &h, sizeof(h));
    *ptr = p;
    return FSDP_OK;
}

int fsdp_ipc_free(void* ptr) {
    if (ptr == nullptr) return FSDP_EINVAL;
    return cuda_status(cudaFree(ptr));
}

int fsdp_ipc_open(const fsdp_ipc_handle* handle, void** ptr) {
    if (handle == nullptr || ptr == nullptr) return FSDP_EINVAL;
    *ptr = nullptr;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle->bytes, sizeof(h));
    return cuda_status(cudaIpcOpenMemHandle(ptr, h, cudaIpcMemLazyEnablePeerAccess));
}

int fsdp_ipc_close(void* ptr) {
    if (ptr == nullptr) return FSDP_EINVAL;
    return cuda_status(cudaIpcCloseMemHandle(ptr));
}

}  // extern "C"
