// fsdpk_api.cu -- host side of libfsdpk.so: the parameter-group plan and the
// extern "C" entry points declared in include/fsdpk.h.
//
// The plan restates the Shard(0) placement of "Sharded Training: FSDP2,
// DTensor, Tensor and Pipeline Parallelism" (fully_shard paragraph): rank r
// keeps chunk r of torch.chunk(param, N, dim=0), i.e. rows
// [r*c, r*c + v_r) with c = ceil(d0 / N), and every rank's shard is padded
// to c rows.  One call = one parameter group = one communication unit.
//
// Everything that can be decided once per group is decided here, on the
// host, and uploaded once: the work units of the segment kernels and the pad
// intervals of the copy-in.  The data calls then only validate pointers and
// launch.
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <new>
#include <vector>

#include "fsdpk.h"
#include "fsdpk_internal.h"

using fsdpk::Interval;
using fsdpk::TileRange;
using fsdpk::Unit;
using fsdpk::FlatSeg;
using fsdpk::kFlatCopyOutShare;
using fsdpk::kFlatMaxElems;
using fsdpk::kFlatMinUnits;
using fsdpk::kFlatPad;

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
    g_last_cuda_error = (int)e;
    return FSDP_ECUDA;
}

bool mul_ok(int64_t a, int64_t b, int64_t* out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > std::numeric_limits<int64_t>::max() / a) return false;
    *out = a * b;
    return true;
}

bool add_ok(int64_t a, int64_t b, int64_t* out) {
    if (b > std::numeric_limits<int64_t>::max() - a) return false;
    *out = a + b;
    return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Split [pos, pos+len) of a (rank, parameter) run into units of at most
// kUnitElems elements.
void push_units(std::vector<Unit>& out, std::vector<int32_t>& out_param, int32_t param,
                int64_t shard_pos, int64_t arena_pos, int64_t len, int32_t is_pad) {
    for (int64_t done = 0; done < len; done += fsdpk::kUnitElems) {
        const int64_t l = std::min<int64_t>(fsdpk::kUnitElems, len - done);
        out.push_back(Unit{shard_pos + done, is_pad ? 0 : arena_pos + done, (int32_t)l, is_pad});
        out_param.push_back(param);
    }
}

// Check the current device is the plan's device.
int check_device(const fsdp_group* g) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    return dev == g->device ? FSDP_OK : FSDP_ESTATE;
}

}  // namespace

namespace {

// AdamW hyper-parameters -> the per-step scalars (binary64 on the host).
bool adam_scalars(const fsdp_adamw_hparams* hp, fsdpk::AdamScalars* sc) {
    if (!(hp->step >= 1) || !(hp->lr >= 0.0) || !(hp->beta1 >= 0.0 && hp->beta1 < 1.0) ||
        !(hp->beta2 >= 0.0 && hp->beta2 < 1.0) || !(hp->eps > 0.0) ||
        !std::isfinite(hp->weight_decay) || !std::isfinite(hp->lr))
        return false;
    const double t = (double)hp->step;
    const double bc1 = 1.0 - std::pow(hp->beta1, t);
    const double bc2 = 1.0 - std::pow(hp->beta2, t);
    sc->decay = (float)(1.0 - hp->lr * hp->weight_decay);
    sc->beta1 = (float)hp->beta1;
    sc->omb1 = (float)(1.0 - hp->beta1);
    sc->beta2 = (float)hp->beta2;
    sc->omb2 = (float)(1.0 - hp->beta2);
    sc->step_size = (float)(hp->lr / bc1);
    sc->inv_bc2_sqrt = (float)(1.0 / std::sqrt(bc2));
    sc->eps = (float)hp->eps;
    return true;
}

}  // namespace

namespace fsdpk {

// The work tables of the virtual ranks [r0, r1), in the local index space
// [(r1 - r0)][S] of buffers that hold only those ranks' shards: real units of
// every (rank j, parameter i), then pad units, the merged pad intervals and
// the copy-in tile ranges.  Reads the per-parameter tables of g.
// Packs of consecutive units [b, e): up to kPackUnits units and kPackElems
// elements each (a single longer unit makes a pack of its own); out receives
// the pack boundaries, out[0] = b and out.back() = e.
void make_packs(const fsdp_group& g, int64_t b, int64_t e, std::vector<int32_t>* out) {
    out->clear();
    for (int64_t k = b; k < e;) {
        out->push_back((int32_t)k);
        int64_t elems = 0, cnt = 0;
        while (k < e && cnt < fsdpk::kPackUnits &&
               (cnt == 0 || elems + g.units[(size_t)k].len <= fsdpk::kPackElems)) {
            elems += g.units[(size_t)k].len;
            ++cnt;
            ++k;
        }
    }
    out->push_back((int32_t)e);
}

// Segments of a flat index space [0, end) from its runs (start, len, code),
// sorted here; the space between runs gets kFlatPad.  Adjacent ranges with
// one code merge, and a sentinel closes the table.
std::vector<FlatSeg> flat_segments(std::vector<std::array<int64_t, 3>> runs, int64_t end) {
    std::sort(runs.begin(), runs.end());
    std::vector<FlatSeg> segs;
    auto put = [&](int64_t start, int32_t code) {
        if (segs.empty() || segs.back().code != code) segs.push_back(FlatSeg{(int32_t)start, code});
    };
    int64_t at = 0;
    for (const auto& r : runs) {
        if (r[1] <= 0) continue;
        if (r[0] > at) put(at, kFlatPad);
        put(r[0], (int32_t)r[2]);
        at = r[0] + r[1];
    }
    if (at < end) put(at, kFlatPad);
    segs.push_back(FlatSeg{(int32_t)end, kFlatPad});
    return segs;
}

// One code per 8-element vector of [0, end) over its segments: the segment's
// code when one segment holds all 8 elements, else 2 m + 1 for entry m of the
// mixed list (mixq: the vector; mixc: its 8 elements' codes, kFlatPad past
// the end).
std::vector<int32_t> flat_codes(const std::vector<FlatSeg>& segs, int64_t end,
                                std::vector<int32_t>* mixq, std::vector<int32_t>* mixc) {
    std::vector<int32_t> codes((size_t)((end + 7) / 8));
    mixq->clear();
    mixc->clear();
    size_t i = 0;
    for (size_t q = 0; q < codes.size(); ++q) {
        const int64_t lo = 8 * (int64_t)q, hi = lo + 8;
        while (segs[i + 1].start <= lo) ++i;
        if (hi <= end && segs[i + 1].start >= hi) {
            codes[q] = segs[i].code;
            continue;
        }
        codes[q] = (int32_t)(2 * mixq->size() + 1);
        mixq->push_back((int32_t)q);
        size_t t = i;
        for (int64_t k = lo; k < hi; ++k) {
            while (k < end && segs[t + 1].start <= k) ++t;
            mixc->push_back(k < end ? segs[t].code : kFlatPad);
        }
    }
    return codes;
}

// The flat path's tables, for a plan of all N ranks with at least
// kFlatMinUnits short and pad units and both index spaces within the codes'
// range; otherwise g->flat stays false.  Shard side: the real units (code
// 2 * (arena_pos - shard_pos)) and the pad units over [N][S].  Arena side,
// when the short runs hold enough of the elements for the flat copy-out: the
// real units (code 2 * (shard_pos - arena_pos)) over [P_arena], the
// alignment gaps between parameters as kFlatPad.
void build_flat_maps(fsdp_group* g) {
    g->flat = false;
    g->flat_copy_out = false;
    for (auto* v : {&g->smap, &g->amap, &g->smixq, &g->amixq, &g->smixc, &g->amixc}) v->clear();
    g->ssegs.clear();
    g->asegs.clear();
    const int64_t LS = (int64_t)g->L * g->S;
    const int64_t n_small = (int64_t)g->units.size() - g->n_long_units;
    if (g->L != g->N || n_small < kFlatMinUnits || LS > kFlatMaxElems ||
        g->P_arena > kFlatMaxElems)
        return;
    std::vector<std::array<int64_t, 3>> sruns, aruns;
    sruns.reserve(g->units.size());
    aruns.reserve((size_t)g->n_real_units);
    int64_t short_elems = 0;
    for (int64_t k = g->n_long_units; k < g->n_real_units; ++k) short_elems += g->units[(size_t)k].len;
    for (const Unit& u : g->units) {
        if (u.is_pad) {
            sruns.push_back({u.shard_pos, u.len, kFlatPad});
        } else {
            sruns.push_back({u.shard_pos, u.len, 2 * (u.arena_pos - u.shard_pos)});
            aruns.push_back({u.arena_pos, u.len, 2 * (u.shard_pos - u.arena_pos)});
        }
    }
    g->ssegs = flat_segments(std::move(sruns), LS);
    g->smap = flat_codes(g->ssegs, LS, &g->smixq, &g->smixc);
    g->flat = true;
    if (short_elems * kFlatCopyOutShare >= g->P) {
        g->asegs = flat_segments(std::move(aruns), g->P_arena);
        g->amap = flat_codes(g->asegs, g->P_arena, &g->amixq, &g->amixc);
        g->flat_copy_out = true;
    }
}

int build_rank_tables(fsdp_group* g, int64_t r0, int64_t r1) {
    const int64_t S = g->S;
    const int32_t n_params = g->n;
    g->units.clear();
    g->unit_param.clear();
    g->intervals.clear();
    g->tile_ranges.clear();
    try {
        for (int64_t j = r0; j < r1; ++j)
            for (int32_t i = 0; i < n_params; ++i) {
                const int64_t v = std::clamp<int64_t>(g->d0[i] - j * g->c[i], 0, g->c[i]);
                push_units(g->units, g->unit_param, i, (j - r0) * S + g->off[i],
                           g->u[i] + j * g->c[i] * g->cols[i], v * g->cols[i], 0);
            }
        g->n_real_units = (int64_t)g->units.size();
        // long real units first (a CTA each in the copy-outs), then the short
        // ones, in packs
        std::vector<size_t> order((size_t)g->n_real_units);
        for (size_t k = 0; k < order.size(); ++k) order[k] = k;
        std::stable_partition(order.begin(), order.end(), [&](size_t k) {
            return g->units[k].len >= fsdpk::kShortRun;
        });
        std::vector<Unit> ru(order.size());
        std::vector<int32_t> rp(order.size());
        for (size_t k = 0; k < order.size(); ++k) {
            ru[k] = g->units[order[k]];
            rp[k] = g->unit_param[order[k]];
        }
        std::copy(ru.begin(), ru.end(), g->units.begin());
        std::copy(rp.begin(), rp.end(), g->unit_param.begin());
        g->n_long_units = 0;
        while (g->n_long_units < g->n_real_units &&
               g->units[(size_t)g->n_long_units].len >= fsdpk::kShortRun)
            ++g->n_long_units;
        make_packs(*g, g->n_long_units, g->n_real_units, &g->packs);
        for (int64_t j = r0; j < r1; ++j)
            for (int32_t i = 0; i < n_params; ++i) {
                const int64_t v = std::clamp<int64_t>(g->d0[i] - j * g->c[i], 0, g->c[i]);
                const int64_t lo = (j - r0) * S + g->off[i] + v * g->cols[i];
                const int64_t len = (g->c[i] - v) * g->cols[i];
                push_units(g->units, g->unit_param, i, lo, 0, len, 1);
                if (len > 0) {
                    if (!g->intervals.empty() && g->intervals.back().hi == lo)
                        g->intervals.back().hi = lo + len;  // merge adjacent pads
                    else
                        g->intervals.push_back(Interval{lo, lo + len});
                }
            }
        make_packs(*g, g->n_long_units, (int64_t)g->units.size(), &g->rpacks);
        if (g->intervals.size() > (size_t)std::numeric_limits<int32_t>::max()) return FSDP_EINVAL;
        const int64_t NS = (r1 - r0) * S;
        g->n_tiles = (NS + fsdpk::kCopyInTile - 1) / fsdpk::kCopyInTile;
        if (!g->intervals.empty()) {
            g->tile_ranges.resize((size_t)g->n_tiles);
            size_t a = 0, b = 0;
            for (int64_t t = 0; t < g->n_tiles; ++t) {
                const int64_t lo = t * fsdpk::kCopyInTile;
                const int64_t hi = lo + fsdpk::kCopyInTile;
                while (a < g->intervals.size() && g->intervals[a].hi <= lo) ++a;
                if (b < a) b = a;
                while (b < g->intervals.size() && g->intervals[b].lo < hi) ++b;
                g->tile_ranges[(size_t)t] = TileRange{(int32_t)a, (int32_t)b};
            }
        }
        if (r0 == 0 && r1 == g->N) build_flat_maps(g);
    } catch (...) {
        return FSDP_ENOMEM;
    }
    return FSDP_OK;
}

// One device allocation for the work tables of g, uploaded once; records the
// current device and its SM count.
int upload_tables(fsdp_group* g) {
    cudaError_t e = cudaGetDevice(&g->device);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(&g->sm_count, cudaDevAttrMultiProcessorCount, g->device);
    if (e != cudaSuccess) return cuda_fail(e);
    struct Table {
        const void* host;
        size_t bytes;
        const void** dev;
    };
    auto table = [](const auto& v, const void** dev) {
        return Table{v.data(), v.size() * sizeof(v[0]), dev};
    };
    const Table tables[] = {
        table(g->units, reinterpret_cast<const void**>(&g->d_units)),
        table(g->intervals, reinterpret_cast<const void**>(&g->d_intervals)),
        table(g->tile_ranges, reinterpret_cast<const void**>(&g->d_tile_ranges)),
        table(g->unit_param, reinterpret_cast<const void**>(&g->d_unit_param)),
        table(g->packs, reinterpret_cast<const void**>(&g->d_packs)),
        table(g->rpacks, reinterpret_cast<const void**>(&g->d_rpacks)),
        table(g->smap, reinterpret_cast<const void**>(&g->d_smap)),
        table(g->smixq, reinterpret_cast<const void**>(&g->d_smixq)),
        table(g->smixc, reinterpret_cast<const void**>(&g->d_smixc)),
        table(g->amap, reinterpret_cast<const void**>(&g->d_amap)),
        table(g->amixq, reinterpret_cast<const void**>(&g->d_amixq)),
        table(g->amixc, reinterpret_cast<const void**>(&g->d_amixc)),
    };
    auto up256 = [](size_t x) { return (x + 255) / 256 * 256; };
    size_t total = 0;
    for (const Table& t : tables) total += up256(t.bytes);
    if (total == 0) return FSDP_OK;
    e = cudaMalloc(&g->dev_mem, total);
    if (e != cudaSuccess) {
        cudaGetLastError();
        g->dev_mem = nullptr;
        return e == cudaErrorMemoryAllocation ? FSDP_ENOMEM : cuda_fail(e);
    }
    char* at = static_cast<char*>(g->dev_mem);
    for (const Table& t : tables) {
        *t.dev = at;
        if (e == cudaSuccess && t.bytes)
            e = cudaMemcpy(at, t.host, t.bytes, cudaMemcpyHostToDevice);
        at += up256(t.bytes);
    }
    if (e != cudaSuccess) {
        cudaFree(g->dev_mem);
        g->dev_mem = nullptr;
        return cuda_fail(e);
    }
    return FSDP_OK;
}

void free_tables(fsdp_group* g) {
    if (g->dev_mem == nullptr) return;
    int prev = -1;
    bool switched = false;
    if (cudaGetDevice(&prev) == cudaSuccess && prev != g->device)
        switched = cudaSetDevice(g->device) == cudaSuccess;
    cudaFree(g->dev_mem);
    g->dev_mem = nullptr;
    if (switched) cudaSetDevice(prev);
}

int record_cuda_error(cudaError_t e) { return cuda_fail(e); }

int check_plan_device(const fsdp_group* g) { return check_device(g); }

bool host_adam_scalars(const fsdp_adamw_hparams* hp, AdamScalars* sc) {
    return adam_scalars(hp, sc);
}

// Debug build: the caller's error words and the test-only narrowing of every
// launch's extents (so that a check can be seen to fire on valid tables).
namespace {
uint32_t* g_debug_words = nullptr;
int64_t g_debug_shrink = 0;
}  // namespace

DebugBounds debug_bounds_raw(int64_t ns, int64_t arena, int32_t kernel, int64_t n_aux) {
    DebugBounds b;
    b.ns = ns - g_debug_shrink;
    b.arena = arena - g_debug_shrink;
    b.n_aux = n_aux;
    b.words = g_debug_words;
    b.kernel = kernel;
    return b;
}

DebugBounds debug_bounds(const fsdp_group& g, int32_t kernel, int64_t n_aux) {
    return debug_bounds_raw((int64_t)g.L * g.S, g.P_arena, kernel, n_aux);
}

}  // namespace fsdpk

extern "C" {


int fsdp_abi_version(void) { return FSDP_ABI_VERSION; }

int fsdp_debug_build(void) {
#ifdef FSDPK_DEBUG
    return 1;
#else
    return 0;
#endif
}

int fsdp_debug_set_error_words(uint32_t* words, int64_t shrink) {
#ifdef FSDPK_DEBUG
    if (shrink < 0) return FSDP_EINVAL;
    if (words != nullptr && (reinterpret_cast<uintptr_t>(words) & 3u) != 0) return FSDP_EALIGN;
    fsdpk::g_debug_words = words;
    fsdpk::g_debug_shrink = shrink;
    return FSDP_OK;
#else
    (void)words;
    (void)shrink;
    return FSDP_ESTATE;
#endif
}

int fsdp_last_cuda_error(void) { return g_last_cuda_error; }

const char* fsdp_status_string(int status) {
    switch (status) {
        case FSDP_OK: return "ok";
        case FSDP_EINVAL: return "invalid argument";
        case FSDP_ENOMEM: return "out of memory";
        case FSDP_ECUDA: return "CUDA error";
        case FSDP_EALIGN: return "pointer not 16-byte aligned";
        case FSDP_ESTATE: return "call not valid in this state (plan of another device, host-only plan, or a capturing stream)";
        default: return "unknown status";
    }
}

namespace {

// The per-parameter tables and the work tables of all N ranks, on the host.
int plan_on_host(const fsdp_param_desc* params, int32_t n_params, int32_t world_size,
                 fsdp_group_t* out) {
    if (out == nullptr) return FSDP_EINVAL;
    *out = nullptr;
    if (n_params < 0 || (n_params > 0 && params == nullptr)) return FSDP_EINVAL;
    if (world_size < 1 || world_size > FSDP_MAX_WORLD) return FSDP_EINVAL;

    fsdp_group* g = new (std::nothrow) fsdp_group();
    if (g == nullptr) return FSDP_ENOMEM;
    auto fail = [&](int st) {
        delete g;
        return st;
    };
    const int64_t N = world_size;
    g->N = world_size;
    g->n = n_params;
    try {
        g->d0.resize(n_params);
        g->cols.resize(n_params);
        g->c.resize(n_params);
        g->s.resize(n_params);
        g->off.resize(n_params);
        g->u.resize(n_params);
    } catch (...) {
        return fail(FSDP_ENOMEM);
    }

    // per-parameter tables
    int64_t S = 0, P = 0, A = 0;
    for (int32_t i = 0; i < n_params; ++i) {
        const fsdp_param_desc& d = params[i];
        if (d.ndim < 0 || d.ndim > FSDP_MAX_NDIM) return fail(FSDP_EINVAL);
        int64_t d0 = 1, cols = 1;
        for (int k = 0; k < d.ndim; ++k) {
            if (d.shape[k] < 0) return fail(FSDP_EINVAL);
            if (k == 0) d0 = d.shape[0];
            else if (!mul_ok(cols, d.shape[k], &cols)) return fail(FSDP_EINVAL);
        }
        const int64_t c = d0 == 0 ? 0 : (d0 + N - 1) / N;  // torch.chunk rows
        int64_t s, numel;
        if (!mul_ok(c, cols, &s) || !mul_ok(d0, cols, &numel)) return fail(FSDP_EINVAL);
        g->d0[i] = d0;
        g->cols[i] = cols;
        g->c[i] = c;
        g->s[i] = s;
        g->off[i] = S;
        if (!add_ok(S, s, &S) || !add_ok(P, numel, &P)) return fail(FSDP_EINVAL);
        // arena: each parameter starts on a multiple of 8 elements (16 bytes)
        int64_t ui;
        if (!add_ok(A, 7, &ui)) return fail(FSDP_EINVAL);
        ui = ui / 8 * 8;
        g->u[i] = ui;
        if (!add_ok(ui, numel, &A)) return fail(FSDP_EINVAL);
    }
    int64_t Aup;
    if (!add_ok(A, 7, &Aup)) return fail(FSDP_EINVAL);
    g->S = S;
    g->P = P;
    g->P_arena = Aup / 8 * 8;
    // every buffer size the data calls imply must fit int64 indexing
    int64_t NS, NA, NNS, tmp;
    if (!mul_ok(N, S, &NS) || !mul_ok(N, g->P_arena, &NA) || !mul_ok(NS, N, &NNS) ||
        !mul_ok(NNS, 4, &tmp) || !mul_ok(NA, 2, &tmp))
        return fail(FSDP_EINVAL);
    if (NS / fsdpk::kCopyInTile + 1 > std::numeric_limits<int32_t>::max()) return fail(FSDP_EINVAL);
    g->pad_elems = NS - P;

    g->L = world_size;
    int st = fsdpk::build_rank_tables(g, 0, N);
    if (st != FSDP_OK) return fail(st);
    *out = g;
    return FSDP_OK;
}

// Every check the data calls rely on, over the host copies of the work
// tables: the extents of every unit, exact coverage of [L][S] by the units,
// each real unit's arena position recomputed from its shard position (the
// Shard(0) placement), the pad intervals against the pad units, and each
// copy-in tile's interval range.  Returns the number of violations.
// The flat path's segments, codes and mixed list of one index space
// [0, end) against its runs (start, len, code): segments strictly increasing
// from 0 with a sentinel at end and no two neighbours with one code; each run
// inside a single segment of its code; as many elements in segments of real
// codes as in real runs (so the rest is kFlatPad); each vector's code pure
// exactly when one segment holds all 8 of its elements, else the next entry
// of the mixed list, which names the vector and each element's code.
int64_t check_flat_space(const std::vector<FlatSeg>& segs, const std::vector<int32_t>& codes,
                         const std::vector<int32_t>& mixq, const std::vector<int32_t>& mixc,
                         const std::vector<std::array<int64_t, 3>>& runs, int64_t end) {
    int64_t bad = 0;
    if (segs.size() < 2 || segs.front().start != 0 || segs.back().start != end ||
        segs.back().code != kFlatPad)
        return 1;
    int64_t real = 0;
    for (size_t i = 0; i + 1 < segs.size(); ++i) {
        if (segs[i + 1].start <= segs[i].start) ++bad;
        if (i + 2 < segs.size() && segs[i + 1].code == segs[i].code) ++bad;
        if (segs[i].code != kFlatPad) {
            if (segs[i].code & 1) ++bad;
            real += (int64_t)segs[i + 1].start - segs[i].start;
        }
    }
    if (bad) return bad;
    auto seg_of = [&](int64_t k) {  // the segment holding element k < end
        size_t lo = 0, hi = segs.size() - 1;
        while (hi - lo > 1) {
            const size_t mid = (lo + hi) / 2;
            if (segs[mid].start <= k) lo = mid; else hi = mid;
        }
        return lo;
    };
    int64_t real_runs = 0;
    for (const auto& r : runs) {
        if (r[1] <= 0) continue;
        if (r[0] < 0 || r[0] + r[1] > end) {
            ++bad;
            continue;
        }
        const size_t i = seg_of(r[0]);
        if (segs[i].code != (int32_t)r[2] || segs[i + 1].start < r[0] + r[1]) ++bad;
        if (r[2] != kFlatPad) real_runs += r[1];
    }
    if (real != real_runs) ++bad;
    if ((int64_t)codes.size() != (end + 7) / 8 || mixc.size() != 8 * mixq.size()) return bad + 1;
    size_t m = 0;
    for (size_t q = 0; q < codes.size(); ++q) {
        const int64_t lo = 8 * (int64_t)q, hi = lo + 8;
        const size_t i = seg_of(lo);
        const bool pure = hi <= end && segs[i + 1].start >= hi;
        if (pure) {
            if (codes[q] != segs[i].code) ++bad;
            continue;
        }
        if (codes[q] != (int32_t)(2 * m + 1) || m >= mixq.size() || mixq[m] != (int32_t)q) {
            ++bad;
            continue;
        }
        for (int e = 0; e < 8; ++e) {
            const int64_t k = lo + e;
            const int32_t want = k < end ? segs[seg_of(k)].code : kFlatPad;
            if (mixc[8 * m + (size_t)e] != want) ++bad;
        }
        ++m;
    }
    if (m != mixq.size()) ++bad;
    return bad;
}

// The flat path of g: built exactly when the plan qualifies, and both
// spaces' tables recomputed from the units.
int64_t check_flat(const fsdp_group& g) {
    const int64_t LS = (int64_t)g.L * g.S;
    const int64_t n_small = (int64_t)g.units.size() - g.n_long_units;
    const bool want = g.L == g.N && n_small >= kFlatMinUnits && LS <= kFlatMaxElems &&
                      g.P_arena <= kFlatMaxElems;
    if (want != g.flat) return 1;
    int64_t short_elems = 0;
    for (int64_t k = g.n_long_units; k < g.n_real_units && k < (int64_t)g.units.size(); ++k)
        short_elems += g.units[(size_t)k].len;
    const bool want_copy_out = want && short_elems * kFlatCopyOutShare >= g.P;
    if (want_copy_out != g.flat_copy_out) return 1;
    const bool arena_empty = g.amap.empty() && g.amixq.empty() && g.amixc.empty() && g.asegs.empty();
    if (!g.flat)
        return (g.smap.empty() && g.smixq.empty() && g.smixc.empty() && g.ssegs.empty() &&
                arena_empty)
                   ? 0
                   : 1;
    std::vector<std::array<int64_t, 3>> sruns, aruns;
    for (const Unit& u : g.units) {
        sruns.push_back({u.shard_pos, u.len,
                         u.is_pad ? (int64_t)kFlatPad : 2 * (u.arena_pos - u.shard_pos)});
        if (!u.is_pad) aruns.push_back({u.arena_pos, u.len, -2 * (u.arena_pos - u.shard_pos)});
    }
    const int64_t bad = check_flat_space(g.ssegs, g.smap, g.smixq, g.smixc, sruns, LS);
    if (!g.flat_copy_out) return bad + (arena_empty ? 0 : 1);
    return bad + check_flat_space(g.asegs, g.amap, g.amixq, g.amixc, aruns, g.P_arena);
}

int64_t check_tables(const fsdp_group& g) {
    int64_t bad = 0;
    const int64_t LS = (int64_t)g.L * g.S;
    const int64_t r0 = 0;  // a group plan holds the ranks [0, N)
    std::vector<std::pair<int64_t, int64_t>> spans;  // (shard_pos, len)
    int64_t pad_elems = 0;
    if (g.unit_param.size() != g.units.size()) ++bad;
    for (size_t k = 0; k < g.units.size(); ++k) {
        const Unit& u = g.units[k];
        const int32_t i = k < g.unit_param.size() ? g.unit_param[k] : -1;
        if (u.len < 1 || u.len > fsdpk::kUnitElems || u.shard_pos < 0 || u.shard_pos + u.len > LS ||
            i < 0 || i >= g.n) {
            ++bad;
            continue;
        }
        if ((k < (size_t)g.n_real_units) == (u.is_pad != 0)) ++bad;  // real units first
        spans.emplace_back(u.shard_pos, u.len);
        // the unit lies inside parameter i's padded shard of its rank
        const int64_t j = u.shard_pos / g.S + r0;
        const int64_t e0 = u.shard_pos - (j - r0) * g.S - g.off[i];
        const int64_t valid = std::clamp<int64_t>(g.d0[i] - j * g.c[i], 0, g.c[i]) * g.cols[i];
        if (e0 < 0 || e0 + u.len > g.s[i]) {
            ++bad;
            continue;
        }
        if (u.is_pad) {
            pad_elems += u.len;
            if (u.arena_pos != 0 || e0 < valid) ++bad;  // pad rows follow the valid rows
        } else {
            if (e0 + u.len > valid) ++bad;
            // rank j's rows of parameter i start at u_i + j * c_i * cols_i in the arena
            if (u.arena_pos != g.u[i] + j * g.c[i] * g.cols[i] + e0) ++bad;
            if (u.arena_pos < 0 || u.arena_pos + u.len > g.P_arena) ++bad;
        }
    }
    // long real units first, then the short ones in packs that cover them
    if (g.n_long_units < 0 || g.n_long_units > g.n_real_units) ++bad;
    for (int64_t k = 0; k < g.n_real_units && k < (int64_t)g.units.size(); ++k)
        if ((g.units[(size_t)k].len >= fsdpk::kShortRun) != (k < g.n_long_units)) ++bad;
    if (g.packs.empty() || g.packs.front() != g.n_long_units || g.packs.back() != g.n_real_units)
        ++bad;
    for (size_t p = 0; p + 1 < g.packs.size(); ++p) {
        const int64_t cnt = (int64_t)g.packs[p + 1] - g.packs[p];
        if (cnt < 1 || cnt > fsdpk::kPackUnits) ++bad;
    }
    // the reduce-scatter's packs cover every unit after the long ones
    if (g.rpacks.empty() || g.rpacks.front() != g.n_long_units ||
        g.rpacks.back() != (int64_t)g.units.size())
        ++bad;
    for (size_t p = 0; p + 1 < g.rpacks.size(); ++p) {
        const int64_t cnt = (int64_t)g.rpacks[p + 1] - g.rpacks[p];
        if (cnt < 1 || cnt > fsdpk::kPackUnits) ++bad;
    }
    std::sort(spans.begin(), spans.end());
    int64_t at = 0;
    for (const auto& sp : spans) {
        if (sp.first != at) ++bad;  // a gap or an overlap in the coverage of [L][S]
        at = sp.first + sp.second;
    }
    if (at != LS) ++bad;
    // pad intervals: sorted, disjoint, inside [L][S], as many elements as the pad units
    int64_t iv_elems = 0, prev_hi = -1;
    for (const Interval& iv : g.intervals) {
        if (iv.lo < 0 || iv.hi > LS || iv.lo >= iv.hi || iv.lo <= prev_hi) ++bad;
        iv_elems += iv.hi - iv.lo;
        prev_hi = iv.hi;
    }
    if (iv_elems != pad_elems || (g.L == g.N && pad_elems != LS - g.P)) ++bad;
    // copy-in tiles: each tile's range holds exactly the intervals that meet it
    if (!g.intervals.empty()) {
        if ((int64_t)g.tile_ranges.size() != g.n_tiles) ++bad;
        for (int64_t t = 0; t < (int64_t)g.tile_ranges.size(); ++t) {
            const int64_t lo = t * fsdpk::kCopyInTile, hi = lo + fsdpk::kCopyInTile;
            const TileRange& tr = g.tile_ranges[(size_t)t];
            for (int32_t q = 0; q < (int32_t)g.intervals.size(); ++q) {
                const bool meets = g.intervals[(size_t)q].lo < hi && g.intervals[(size_t)q].hi > lo;
                const bool inside = q >= tr.begin && q < tr.end;
                if (meets != inside) ++bad;
            }
        }
    }
    bad += check_flat(g);
    return bad;
}

}  // namespace

int fsdp_plan_group(const fsdp_param_desc* params, int32_t n_params, int32_t world_size,
                    fsdp_group_t* out) {
    int st = plan_on_host(params, n_params, world_size, out);
    if (st != FSDP_OK) return st;
    st = fsdpk::upload_tables(*out);
    if (st != FSDP_OK) {
        delete *out;
        *out = nullptr;
    }
    return st;
}

int fsdp_plan_group_host(const fsdp_param_desc* params, int32_t n_params, int32_t world_size,
                         fsdp_group_t* out) {
    return plan_on_host(params, n_params, world_size, out);
}

int fsdp_group_check(fsdp_group_t g, int64_t* violations) {
    if (g == nullptr || violations == nullptr) return FSDP_EINVAL;
    *violations = check_tables(*g);
    return FSDP_OK;
}

int fsdp_group_flat(fsdp_group_t g, int32_t* flat, int64_t* mixed_shard, int64_t* mixed_arena) {
    if (g == nullptr) return FSDP_EINVAL;
    if (flat) *flat = (g->flat ? 1 : 0) | (g->flat_copy_out ? 2 : 0);
    if (mixed_shard) *mixed_shard = (int64_t)g->smixq.size();
    if (mixed_arena) *mixed_arena = (int64_t)g->amixq.size();
    return FSDP_OK;
}

int fsdp_group_sizes(fsdp_group_t g, int64_t* S, int64_t* P, int64_t* P_arena) {
    if (g == nullptr) return FSDP_EINVAL;
    if (S) *S = g->S;
    if (P) *P = g->P;
    if (P_arena) *P_arena = g->P_arena;
    return FSDP_OK;
}

int fsdp_group_param_offsets(fsdp_group_t g, int64_t* shard_off, int64_t* arena_off,
                             int64_t* chunk_rows) {
    if (g == nullptr) return FSDP_EINVAL;
    for (int32_t i = 0; i < g->n; ++i) {
        if (shard_off) shard_off[i] = g->off[i];
        if (arena_off) arena_off[i] = g->u[i];
        if (chunk_rows) chunk_rows[i] = g->c[i];
    }
    return FSDP_OK;
}

void fsdp_destroy_group(fsdp_group_t g) {
    if (g == nullptr) return;
    fsdpk::free_tables(g);
    delete g;
}

int fsdp_shard_params(fsdp_group_t g, const float* full_arena, float* master,
                      fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if ((int64_t)g->N * g->S > 0 && master == nullptr) return FSDP_EINVAL;
    if (g->P > 0 && full_arena == nullptr) return FSDP_EINVAL;
    if (!aligned16(full_arena) || !aligned16(master)) return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaError_t e = fsdpk::launch_shard(*g, full_arena, master, (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_copy_in(fsdp_group_t g, const float* master, uint16_t* ag, fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if ((int64_t)g->N * g->S > 0 && (master == nullptr || ag == nullptr)) return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(ag)) return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaError_t e = fsdpk::launch_copy_in(*g, master, ag, (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_copy_out(fsdp_group_t g, const uint16_t* ag, uint16_t* arena, fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if (g->P > 0 && (ag == nullptr || arena == nullptr)) return FSDP_EINVAL;
    if (!aligned16(ag) || !aligned16(arena)) return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaError_t e = fsdpk::launch_copy_out(*g, ag, arena, (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_rs_reduce(fsdp_group_t g, const uint16_t* grads, int32_t op, float* packed_or_null,
                   float* reduced, fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if (op != FSDP_SUM && op != FSDP_AVG && op != FSDP_SUM_THEN_DIV) return FSDP_EINVAL;
    const int64_t NS = (int64_t)g->N * g->S;
    if (NS > 0 && reduced == nullptr) return FSDP_EINVAL;
    if (g->P > 0 && grads == nullptr) return FSDP_EINVAL;
    if (!aligned16(grads) || !aligned16(reduced) || !aligned16(packed_or_null))
        return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (packed_or_null == nullptr) {
        e = fsdpk::launch_rs_fused(*g, grads, op, reduced, s);
    } else {
        // staged: materialise every rank's reduce-scatter input, reduce it,
        // and for SUM_THEN_DIV divide in a separate pass
        e = fsdpk::launch_rs_pack(*g, grads, packed_or_null, s);
        if (e == cudaSuccess)
            e = fsdpk::launch_rs_reduce_packed(*g, packed_or_null, op == FSDP_AVG ? FSDP_AVG : FSDP_SUM,
                                               reduced, s);
        if (e == cudaSuccess && op == FSDP_SUM_THEN_DIV) e = fsdpk::launch_div_inplace(*g, reduced, s);
    }
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_adamw_step(fsdp_group_t g, float* master, float* m, float* v, const float* grad,
                    const fsdp_adamw_hparams* hp, fsdp_stream_t stream) {
    if (g == nullptr || hp == nullptr) return FSDP_EINVAL;
    const int64_t NS = (int64_t)g->N * g->S;
    if (NS > 0 && (master == nullptr || m == nullptr || v == nullptr || grad == nullptr))
        return FSDP_EINVAL;
    fsdpk::AdamScalars sc;
    if (!adam_scalars(hp, &sc)) return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(grad))
        return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaError_t e = fsdpk::launch_adamw(*g, master, m, v, grad, sc, (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_rs_adamw_step(fsdp_group_t g, const uint16_t* grads, int32_t op, float* master,
                       float* m, float* v, const fsdp_adamw_hparams* hp, uint16_t* ag_next,
                       float* reduced, fsdp_stream_t stream) {
    if (g == nullptr || hp == nullptr) return FSDP_EINVAL;
    if (op != FSDP_SUM && op != FSDP_AVG && op != FSDP_SUM_THEN_DIV) return FSDP_EINVAL;
    const int64_t NS = (int64_t)g->N * g->S;
    if (NS > 0 && (master == nullptr || m == nullptr || v == nullptr)) return FSDP_EINVAL;
    if (g->P > 0 && grads == nullptr) return FSDP_EINVAL;
    fsdpk::AdamScalars sc;
    if (!adam_scalars(hp, &sc)) return FSDP_EINVAL;
    if (!aligned16(grads) || !aligned16(master) || !aligned16(m) || !aligned16(v) ||
        !aligned16(ag_next) || !aligned16(reduced))
        return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaError_t e = fsdpk::launch_rs_adamw(*g, grads, op, master, m, v, sc, ag_next, reduced,
                                           (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

namespace {

int group_step(fsdp_group_t g, float* master, float* m, float* v, const uint16_t* grads,
               int32_t op, const fsdpk::AdamScalars& sc, const fsdpk::AdamScalars* sc_dev,
               uint16_t* ag, uint16_t* arena, float* reduced, fsdp_stream_t stream,
               const fsdpk::StepCounter& ctr = fsdpk::StepCounter{}) {
    if (op != FSDP_SUM && op != FSDP_AVG && op != FSDP_SUM_THEN_DIV) return FSDP_EINVAL;
    const int64_t NS = (int64_t)g->N * g->S;
    if (NS > 0 && (master == nullptr || m == nullptr || v == nullptr || ag == nullptr ||
                   reduced == nullptr))
        return FSDP_EINVAL;
    if (g->P > 0 && (grads == nullptr || arena == nullptr)) return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(grads) ||
        !aligned16(ag) || !aligned16(arena) || !aligned16(reduced) || !aligned16(sc_dev))
        return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (NS == 0 && ctr.step != nullptr) {
        // nothing to update, but the step still counts
        e = fsdpk::launch_adamw_prepare(ctr.lr, ctr.beta1, ctr.beta2, ctr.eps, ctr.wd, ctr.step,
                                        ctr.out, s);
    } else if (NS <= FSDP_SMALL_STEP_ELEMS) {
        e = fsdpk::launch_small_step(*g, master, m, v, grads, op, ag, arena, reduced, sc, sc_dev,
                                     s, ctr);
    } else {
        e = cudaSuccess;
        if (ctr.step != nullptr)  // the counter and the scalars first, for the stage kernels
            e = fsdpk::launch_adamw_prepare(ctr.lr, ctr.beta1, ctr.beta2, ctr.eps, ctr.wd,
                                            ctr.step, ctr.out, s);
        if (e == cudaSuccess) e = fsdpk::launch_copy_in(*g, master, ag, s);
        if (e == cudaSuccess) e = fsdpk::launch_copy_out(*g, ag, arena, s);
        if (e == cudaSuccess) e = fsdpk::launch_rs_fused(*g, grads, op, reduced, s);
        if (e == cudaSuccess) e = fsdpk::launch_adamw(*g, master, m, v, reduced, sc, s, sc_dev);
    }
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

}  // namespace

int fsdp_group_step(fsdp_group_t g, float* master, float* m, float* v, const uint16_t* grads,
                    int32_t op, const fsdp_adamw_hparams* hp, uint16_t* ag, uint16_t* arena,
                    float* reduced, fsdp_stream_t stream) {
    if (g == nullptr || hp == nullptr) return FSDP_EINVAL;
    fsdpk::AdamScalars sc;
    if (!adam_scalars(hp, &sc)) return FSDP_EINVAL;
    return group_step(g, master, m, v, grads, op, sc, nullptr, ag, arena, reduced, stream);
}

int fsdp_group_step_dev(fsdp_group_t g, float* master, float* m, float* v,
                        const uint16_t* grads, int32_t op,
                        const fsdp_adamw_dev_scalars* scalars_dev, uint16_t* ag,
                        uint16_t* arena, float* reduced, fsdp_stream_t stream) {
    if (g == nullptr || scalars_dev == nullptr) return FSDP_EINVAL;
    const fsdpk::AdamScalars none{};
    return group_step(g, master, m, v, grads, op, none,
                      reinterpret_cast<const fsdpk::AdamScalars*>(scalars_dev), ag, arena,
                      reduced, stream);
}

int fsdp_group_step_graph(fsdp_group_t g, float* master, float* m, float* v,
                          const uint16_t* grads, int32_t op, const fsdp_adamw_hparams* hp,
                          int64_t* step_dev, fsdp_adamw_dev_scalars* scalars_dev, uint16_t* ag,
                          uint16_t* arena, float* reduced, fsdp_stream_t stream) {
    if (g == nullptr || hp == nullptr || step_dev == nullptr || scalars_dev == nullptr)
        return FSDP_EINVAL;
    fsdp_adamw_hparams probe = *hp;
    probe.step = 1;  // the step comes from step_dev; validate the rest
    fsdpk::AdamScalars unused;
    if (!adam_scalars(&probe, &unused)) return FSDP_EINVAL;
    if ((reinterpret_cast<uintptr_t>(step_dev) & 7u) || !aligned16(scalars_dev))
        return FSDP_EALIGN;
    fsdpk::StepCounter ctr;
    ctr.step = step_dev;
    ctr.out = reinterpret_cast<fsdpk::AdamScalars*>(scalars_dev);
    ctr.lr = hp->lr;
    ctr.beta1 = hp->beta1;
    ctr.beta2 = hp->beta2;
    ctr.eps = hp->eps;
    ctr.wd = hp->weight_decay;
    const int64_t NS = (int64_t)g->N * g->S;
    // the stage kernels of a large group read the scalars the prepare wrote
    const fsdpk::AdamScalars* sc_dev =
        NS <= FSDP_SMALL_STEP_ELEMS ? nullptr : ctr.out;
    return group_step(g, master, m, v, grads, op, fsdpk::AdamScalars{}, sc_dev, ag, arena,
                      reduced, stream, ctr);
}

int fsdp_grad_accumulate(fsdp_group_t g, const uint16_t* grads, float* acc, int32_t first,
                         fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if ((int64_t)g->N * g->P_arena > 0 && (grads == nullptr || acc == nullptr)) return FSDP_EINVAL;
    if (!aligned16(grads) || !aligned16(acc)) return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaError_t e = fsdpk::launch_accumulate(*g, grads, acc, first ? 1 : 0, (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_rs_reduce_accumulated(fsdp_group_t g, const uint16_t* grads_or_null, const float* acc,
                               int32_t op, float* reduced, fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if (op != FSDP_SUM && op != FSDP_AVG && op != FSDP_SUM_THEN_DIV) return FSDP_EINVAL;
    if ((int64_t)g->N * g->S > 0 && reduced == nullptr) return FSDP_EINVAL;
    if (g->P > 0 && acc == nullptr) return FSDP_EINVAL;
    if (!aligned16(grads_or_null) || !aligned16(acc) || !aligned16(reduced)) return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaError_t e = fsdpk::launch_rs_reduce_acc(*g, grads_or_null, acc, op, reduced,
                                                (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_copy_in_fp8(fsdp_group_t g, const float* master, uint8_t* ag8, float* scales,
                     fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if ((int64_t)g->N * g->S > 0 && (master == nullptr || ag8 == nullptr)) return FSDP_EINVAL;
    if (g->n > 0 && scales == nullptr) return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(ag8) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaError_t e = fsdpk::launch_copy_in_fp8(*g, master, ag8, scales, (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_copy_in_fp8_scaled(fsdp_group_t g, const float* master, const float* scales,
                            uint8_t* ag8, fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if ((int64_t)g->N * g->S > 0 && (master == nullptr || ag8 == nullptr)) return FSDP_EINVAL;
    if (g->n > 0 && scales == nullptr) return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(ag8) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaError_t e = fsdpk::launch_copy_in_fp8_scaled(*g, master, ag8, scales, (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_rs_adamw_step_fp8(fsdp_group_t g, const uint16_t* grads, int32_t op, float* master,
                           float* m, float* v, const fsdp_adamw_hparams* hp,
                           const float* scales_prev, uint8_t* ag8_next, float* scales_next,
                           float* reduced, fsdp_stream_t stream) {
    if (g == nullptr || hp == nullptr) return FSDP_EINVAL;
    if (op != FSDP_SUM && op != FSDP_AVG && op != FSDP_SUM_THEN_DIV) return FSDP_EINVAL;
    const int64_t NS = (int64_t)g->N * g->S;
    if (NS > 0 && (master == nullptr || m == nullptr || v == nullptr || ag8_next == nullptr))
        return FSDP_EINVAL;
    if (g->P > 0 && grads == nullptr) return FSDP_EINVAL;
    if (g->n > 0 && (scales_prev == nullptr || scales_next == nullptr)) return FSDP_EINVAL;
    if (scales_prev != nullptr && scales_prev == scales_next) return FSDP_EINVAL;
    fsdpk::AdamScalars sc;
    if (!adam_scalars(hp, &sc)) return FSDP_EINVAL;
    if (!aligned16(grads) || !aligned16(master) || !aligned16(m) || !aligned16(v) ||
        !aligned16(ag8_next) || !aligned16(reduced) ||
        (reinterpret_cast<uintptr_t>(scales_prev) & 3u) ||
        (reinterpret_cast<uintptr_t>(scales_next) & 3u))
        return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    const cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    if (g->n > 0) e = cudaMemsetAsync(scales_next, 0, sizeof(float) * (size_t)g->n, s);
    // scales_next holds the amax bits (non-negative floats order as integers)
    // until the last launch turns them into scales
    if (e == cudaSuccess)
        e = fsdpk::launch_rs_adamw_fp8(*g, grads, op, master, m, v, sc, scales_prev, ag8_next,
                                       reinterpret_cast<unsigned*>(scales_next), reduced, s);
    if (e == cudaSuccess) e = fsdpk::launch_fp8_scales_from_amax(*g, scales_next, s);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_copy_out_fp8(fsdp_group_t g, const uint8_t* ag8, uint8_t* arena8, fsdp_stream_t stream) {
    if (g == nullptr) return FSDP_EINVAL;
    if (g->P > 0 && (ag8 == nullptr || arena8 == nullptr)) return FSDP_EINVAL;
    if (!aligned16(ag8) || !aligned16(arena8)) return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    cudaError_t e = fsdpk::launch_copy_out_fp8(*g, ag8, arena8, (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_adamw_prepare(const fsdp_adamw_hparams* hp, int64_t* step_dev,
                       fsdp_adamw_dev_scalars* scalars_dev, fsdp_stream_t stream) {
    if (hp == nullptr || step_dev == nullptr || scalars_dev == nullptr) return FSDP_EINVAL;
    fsdp_adamw_hparams probe = *hp;
    probe.step = 1;  // the step comes from step_dev; validate the rest
    fsdpk::AdamScalars unused;
    if (!adam_scalars(&probe, &unused)) return FSDP_EINVAL;
    if ((reinterpret_cast<uintptr_t>(step_dev) & 7u) || !aligned16(scalars_dev))
        return FSDP_EALIGN;
    cudaError_t e = fsdpk::launch_adamw_prepare(
        hp->lr, hp->beta1, hp->beta2, hp->eps, hp->weight_decay, step_dev,
        reinterpret_cast<fsdpk::AdamScalars*>(scalars_dev), (cudaStream_t)stream);
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_adamw_step_dev(fsdp_group_t g, float* master, float* m, float* v, const float* grad,
                        const fsdp_adamw_dev_scalars* scalars_dev, fsdp_stream_t stream) {
    if (g == nullptr || scalars_dev == nullptr) return FSDP_EINVAL;
    const int64_t NS = (int64_t)g->N * g->S;
    if (NS > 0 && (master == nullptr || m == nullptr || v == nullptr || grad == nullptr))
        return FSDP_EINVAL;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(grad) ||
        !aligned16(scalars_dev))
        return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    const fsdpk::AdamScalars none{};
    cudaError_t e = fsdpk::launch_adamw(*g, master, m, v, grad, none, (cudaStream_t)stream,
                                        reinterpret_cast<const fsdpk::AdamScalars*>(scalars_dev));
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

int fsdp_rs_adamw_step_dev(fsdp_group_t g, const uint16_t* grads, int32_t op, float* master,
                           float* m, float* v, const fsdp_adamw_dev_scalars* scalars_dev,
                           uint16_t* ag_next, float* reduced, fsdp_stream_t stream) {
    if (g == nullptr || scalars_dev == nullptr) return FSDP_EINVAL;
    if (op != FSDP_SUM && op != FSDP_AVG && op != FSDP_SUM_THEN_DIV) return FSDP_EINVAL;
    const int64_t NS = (int64_t)g->N * g->S;
    if (NS > 0 && (master == nullptr || m == nullptr || v == nullptr)) return FSDP_EINVAL;
    if (g->P > 0 && grads == nullptr) return FSDP_EINVAL;
    if (!aligned16(grads) || !aligned16(master) || !aligned16(m) || !aligned16(v) ||
        !aligned16(ag_next) || !aligned16(reduced) || !aligned16(scalars_dev))
        return FSDP_EALIGN;
    int st = check_device(g);
    if (st != FSDP_OK) return st;
    const fsdpk::AdamScalars none{};
    cudaError_t e = fsdpk::launch_rs_adamw(*g, grads, op, master, m, v, none, ag_next, reduced,
                                           (cudaStream_t)stream,
                                           reinterpret_cast<const fsdpk::AdamScalars*>(scalars_dev));
    return e == cudaSuccess ? FSDP_OK : cuda_fail(e);
}

}  // extern "C"
