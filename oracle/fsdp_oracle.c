/*
 * fsdp_oracle.c -- plain, slow CPU oracle for the FSDP2 per-parameter
 * sharding step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the CPU-baseline leg of the benchmark may load this library.  It shares no
 * code, header, table or helper with the CUDA path: every index below is
 * computed again from the definitions, in the most direct nested loops.
 *
 * Sources (web pages; cited by title and section):
 *   [ML] "Sharded Training: FSDP2, DTensor, Tensor and Pipeline Parallelism"
 *        (mlinterviewnotes course 27) -- the fully_shard paragraph (Shard(0),
 *        torch.chunk, internal padding, one group per call), the "Mixed
 *        precision" paragraph (bf16 all-gather, fp32 reduce), the "Other
 *        controls" paragraph (set_force_sum_reduction_for_comms), the lab's
 *        "The bug Adam hid" paragraph (AVG vs SUM + own division), Fence 1
 *        (2+2+12 accounting), Fence 4 (AdamW after sharding).
 *   [MS] "Introduction to PyTorch FSDP2 Backend Features" -- "Working
 *        Principle" (lifecycle: all-gather, compute, reduce-scatter, update)
 *        and "Mixed Precision" (bf16 compute copy, fp32 gradient reduction).
 *
 * Notation for one parameter group of n parameters over N ranks:
 *   d0_i rows, cols_i = product of the other dims (1 for a 1-D parameter)
 *   c_i   = ceil(d0_i / N)                       torch.chunk chunk rows
 *   v_i,r = clamp(d0_i - r*c_i, 0, c_i)          rank r's real rows
 *   s_i   = c_i*cols_i, off_i = sum_{k<i} s_k, S = sum_i s_i
 *   u_i   = unsharded (arena) offset: each start rounded up to 8 elements
 * Buffers: master/m/v/grad-shard/all-gather are rank-major [N][S]; the
 * unsharded parameters and each rank's full gradients use the arena layout
 * [P_arena] with parameter i at u_i.
 *
 * Compiled with -O2 -ffp-contract=off and no fast-math, so every float
 * operation below is one IEEE-754 binary32 (or binary64) operation, rounded
 * to nearest even.  OpenMP only splits outer loops; each output element is
 * computed by exactly the same sequence of operations in any thread count.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - pad rows are the trailing rows of a rank's shard, value +0;
 *   - the group buffer is rank-major [N][S], parameters in registration order;
 *   - the reduction is a left fold from rank 0 in binary32;
 *   - AVG = (ordered SUM) / N, one binary32 division; SUM_THEN_DIV applies the
 *     same division as a second pass over the SUM output;
 *   - AdamW is PyTorch's documented decoupled-weight-decay AdamW, evaluated
 *     here in binary64 and rounded once to binary32 per stored output;
 *   - fp32 -> bf16 is IEEE round-to-nearest-even on the bit pattern; NaN maps
 *     to a quiet NaN (payload is not part of the contract).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_SUM 0
#define OR_AVG 1
#define OR_SUM_THEN_DIV 2

/* ------------------------------------------------------------------ */
/* threads                                                            */
/* ------------------------------------------------------------------ */
void or_set_threads(int t) {
#ifdef _OPENMP
    if (t > 0) omp_set_num_threads(t);
#else
    (void)t;
#endif
}

int or_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* plan: torch.chunk along dim 0 and the padded shard layout           */
/* [ML] fully_shard paragraph: rank r keeps chunk r of                  */
/* torch.chunk(param, world, dim=0), padded when rows do not divide.   */
/* ------------------------------------------------------------------ */

/* chunk rows used by torch.chunk: ceil(d0 / N); 0 for an empty dim */
int64_t or_chunk_rows(int64_t d0, int32_t N) {
    if (d0 <= 0) return 0;
    return (d0 + N - 1) / N;
}

/* real (unpadded) rows that rank r holds */
int64_t or_valid_rows(int64_t d0, int32_t N, int32_t r) {
    int64_t c = or_chunk_rows(d0, N);
    int64_t left = d0 - (int64_t)r * c;
    if (left < 0) left = 0;
    if (left > c) left = c;
    return left;
}

/*
 * Fill the per-parameter tables.  out_sizes receives {S, P, P_arena}.
 */
void or_plan(const int64_t* d0, const int64_t* cols, int32_t n, int32_t N,
             int64_t* c, int64_t* s, int64_t* off, int64_t* u,
             int64_t* out_sizes) {
    int64_t S = 0, P = 0, A = 0;
    for (int32_t i = 0; i < n; ++i) {
        c[i] = or_chunk_rows(d0[i], N);
        s[i] = c[i] * cols[i];
        off[i] = S;
        S += s[i];
        /* arena start rounded up to a multiple of 8 elements */
        u[i] = ((A + 7) / 8) * 8;
        A = u[i] + d0[i] * cols[i];
        P += d0[i] * cols[i];
    }
    out_sizes[0] = S;
    out_sizes[1] = P;
    out_sizes[2] = ((A + 7) / 8) * 8;
}

/* ------------------------------------------------------------------ */
/* bf16 <-> fp32                                                       */
/* [ML] "Mixed precision": param_dtype bf16 copies are all-gathered;   */
/* [MS] "Mixed Precision": FP32 storage -> cast to BF16.               */
/* ------------------------------------------------------------------ */

/* IEEE round-to-nearest-even from binary32 to bfloat16 (bit pattern). */
uint16_t or_bf16_rne_bits(uint32_t x) {
    uint32_t exp = (x >> 23) & 0xFFu;
    uint32_t man = x & 0x7FFFFFu;
    if (exp == 0xFFu && man != 0) {
        /* NaN: keep the sign, force the quiet bit, keep the top payload */
        return (uint16_t)((x >> 16) | 0x0040u);
    }
    /* Keep the upper 16 bits; look at the 16 dropped bits. */
    uint32_t upper = x >> 16;
    uint32_t dropped = x & 0xFFFFu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (upper & 1u))) {
        upper += 1u; /* carries into the exponent correctly, up to Inf */
    }
    return (uint16_t)upper;
}

float or_bf16_to_f32(uint16_t h) {
    uint32_t x = (uint32_t)h << 16;
    float f;
    memcpy(&f, &x, 4);
    return f;
}

static uint32_t f32_bits(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    return x;
}

void or_cast_bf16(const float* x, uint16_t* y, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k) y[k] = or_bf16_rne_bits(f32_bits(x[k]));
}

void or_cast_bf16_bits(const uint32_t* x, uint16_t* y, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k) y[k] = or_bf16_rne_bits(x[k]);
}

/* ------------------------------------------------------------------ */
/* shard: full fp32 parameters (arena layout) -> padded master [N][S]  */
/* ------------------------------------------------------------------ */
void or_shard(const int64_t* d0, const int64_t* cols, int32_t n, int32_t N,
              const float* full, float* master) {
    int64_t c[n > 0 ? n : 1], s[n > 0 ? n : 1], off[n > 0 ? n : 1],
        u[n > 0 ? n : 1], sz[3];
    or_plan(d0, cols, n, N, c, s, off, u, sz);
    int64_t S = sz[0];
#pragma omp parallel for schedule(static)
    for (int32_t r = 0; r < N; ++r) {
        for (int32_t i = 0; i < n; ++i) {
            for (int64_t row = 0; row < c[i]; ++row) {
                int64_t grow = (int64_t)r * c[i] + row; /* row in the full param */
                for (int64_t col = 0; col < cols[i]; ++col) {
                    int64_t dst = (int64_t)r * S + off[i] + row * cols[i] + col;
                    if (grow < d0[i])
                        master[dst] = full[u[i] + grow * cols[i] + col];
                    else
                        master[dst] = 0.0f; /* pad row */
                }
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* a1 copy-in: fp32 shard -> bf16 slot r of the all-gather buffer      */
/* ------------------------------------------------------------------ */
void or_copy_in(const int64_t* d0, const int64_t* cols, int32_t n, int32_t N,
                const float* master, uint16_t* ag) {
    int64_t c[n > 0 ? n : 1], s[n > 0 ? n : 1], off[n > 0 ? n : 1],
        u[n > 0 ? n : 1], sz[3];
    or_plan(d0, cols, n, N, c, s, off, u, sz);
    int64_t S = sz[0];
#pragma omp parallel for schedule(static)
    for (int32_t r = 0; r < N; ++r) {
        for (int32_t i = 0; i < n; ++i) {
            int64_t v = or_valid_rows(d0[i], N, r);
            for (int64_t row = 0; row < c[i]; ++row) {
                for (int64_t col = 0; col < cols[i]; ++col) {
                    int64_t k = (int64_t)r * S + off[i] + row * cols[i] + col;
                    ag[k] = (row < v) ? or_bf16_rne_bits(f32_bits(master[k]))
                                      : (uint16_t)0; /* +0 in every pad row */
                }
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* a2 copy-out: all-gather buffer -> unsharded per-parameter views     */
/* unsharded_i[row] = slot r = row / c_i, local row row - r*c_i.       */
/* ------------------------------------------------------------------ */
void or_copy_out(const int64_t* d0, const int64_t* cols, int32_t n, int32_t N,
                 const uint16_t* ag, uint16_t* arena) {
    int64_t c[n > 0 ? n : 1], s[n > 0 ? n : 1], off[n > 0 ? n : 1],
        u[n > 0 ? n : 1], sz[3];
    or_plan(d0, cols, n, N, c, s, off, u, sz);
    int64_t S = sz[0];
    for (int32_t i = 0; i < n; ++i) {
#pragma omp parallel for schedule(static)
        for (int64_t row = 0; row < d0[i]; ++row) {
            int64_t r = row / c[i];
            int64_t local = row - r * c[i];
            for (int64_t col = 0; col < cols[i]; ++col)
                arena[u[i] + row * cols[i] + col] =
                    ag[r * S + off[i] + local * cols[i] + col];
        }
    }
}

/* ------------------------------------------------------------------ */
/* a3 reduce-scatter packing (reduce_dtype fp32)                       */
/* packed[src r][dst j][off_i + e] = fp32(grad_r,i[j*c_i*cols_i + e])  */
/* for the real rows of chunk j, +0 for its pad rows.                  */
/* grads: [N][P_arena] bf16; packed: [N][N][S] fp32.                   */
/* ------------------------------------------------------------------ */
void or_pack(const int64_t* d0, const int64_t* cols, int32_t n, int32_t N,
             const uint16_t* grads, float* packed) {
    int64_t c[n > 0 ? n : 1], s[n > 0 ? n : 1], off[n > 0 ? n : 1],
        u[n > 0 ? n : 1], sz[3];
    or_plan(d0, cols, n, N, c, s, off, u, sz);
    int64_t S = sz[0], A = sz[2];
#pragma omp parallel for collapse(2) schedule(static)
    for (int32_t r = 0; r < N; ++r) {
        for (int32_t j = 0; j < N; ++j) {
            for (int32_t i = 0; i < n; ++i) {
                int64_t v = or_valid_rows(d0[i], N, j);
                for (int64_t row = 0; row < c[i]; ++row) {
                    for (int64_t col = 0; col < cols[i]; ++col) {
                        int64_t dst = ((int64_t)r * N + j) * S + off[i] +
                                      row * cols[i] + col;
                        if (row < v) {
                            int64_t grow = (int64_t)j * c[i] + row;
                            packed[dst] = or_bf16_to_f32(
                                grads[(int64_t)r * A + u[i] + grow * cols[i] + col]);
                        } else {
                            packed[dst] = 0.0f;
                        }
                    }
                }
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* a4 reduce: red[j][k] = ((p_0 + p_1) + p_2) + ... + p_{N-1}          */
/* with p_r = packed[r][j][k], each add one binary32 RN add.           */
/* AVG divides once by N; SUM_THEN_DIV runs the same division as a     */
/* separate pass ([ML] "Other controls" and "The bug Adam hid").       */
/* ------------------------------------------------------------------ */
void or_reduce_packed(int32_t N, int64_t S, const float* packed, int32_t op,
                      float* red) {
    int64_t total = (int64_t)N * S;
#pragma omp parallel for schedule(static)
    for (int64_t jk = 0; jk < total; ++jk) {
        float acc = packed[jk]; /* r = 0: packed[0][j][k] */
        for (int32_t r = 1; r < N; ++r) acc = acc + packed[(int64_t)r * total + jk];
        float out = acc;
        if (op == OR_AVG) out = out / (float)N;
        red[jk] = out;
    }
    if (op == OR_SUM_THEN_DIV) {
#pragma omp parallel for schedule(static)
        for (int64_t jk = 0; jk < total; ++jk) red[jk] = red[jk] / (float)N;
    }
}

/* ------------------------------------------------------------------ */
/* a3 + a4 from the same definitions without the packed intermediate:  */
/* red[j][off_i + e] = fold over r of fp32(grad_r,i[j*c_i*cols_i + e]) */
/* for the real rows of chunk j, +0 for its pad rows; then the op.     */
/* Used where [N][N][S] would not fit in host memory.                  */
/* ------------------------------------------------------------------ */
void or_reduce_scatter_direct(const int64_t* d0, const int64_t* cols, int32_t n,
                              int32_t N, const uint16_t* grads, int32_t op,
                              float* red) {
    int64_t c[n > 0 ? n : 1], s[n > 0 ? n : 1], off[n > 0 ? n : 1],
        u[n > 0 ? n : 1], sz[3];
    or_plan(d0, cols, n, N, c, s, off, u, sz);
    int64_t S = sz[0], A = sz[2];
    for (int32_t j = 0; j < N; ++j) {
        for (int32_t i = 0; i < n; ++i) {
            int64_t v = or_valid_rows(d0[i], N, j);
#pragma omp parallel for schedule(static)
            for (int64_t row = 0; row < c[i]; ++row) {
                for (int64_t col = 0; col < cols[i]; ++col) {
                    int64_t dst = (int64_t)j * S + off[i] + row * cols[i] + col;
                    if (row >= v) {
                        red[dst] = 0.0f;
                        continue;
                    }
                    int64_t src = u[i] + ((int64_t)j * c[i] + row) * cols[i] + col;
                    float acc = or_bf16_to_f32(grads[src]);
                    for (int32_t r = 1; r < N; ++r)
                        acc = acc + or_bf16_to_f32(grads[(int64_t)r * A + src]);
                    if (op == OR_AVG) acc = acc / (float)N;
                    red[dst] = acc;
                }
            }
        }
    }
    if (op == OR_SUM_THEN_DIV) {
        int64_t total = (int64_t)N * S;
#pragma omp parallel for schedule(static)
        for (int64_t k = 0; k < total; ++k) red[k] = red[k] / (float)N;
    }
}

/* ------------------------------------------------------------------ */
/* Gradient accumulation without sync ([ML] Other controls:            */
/* set_requires_gradient_sync(False) accumulates the unsharded         */
/* gradients and skips the reduce-scatter).  Accumulated in             */
/* reduce_dtype fp32, a left fold over microbatches:                    */
/*   first: acc[k] = fp32(g[k]);  later: acc[k] = acc[k] + fp32(g[k])   */
/* over every element of the per-rank arenas [N][P_arena].              */
/* ------------------------------------------------------------------ */
void or_accumulate(float* acc, const uint16_t* grads, int64_t count, int32_t first) {
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < count; ++k) {
        float g = or_bf16_to_f32(grads[k]);
        acc[k] = first ? g : acc[k] + g;
    }
}

/* Reduce-scatter of fp32 per-rank arenas [N][P_arena] (the accumulated
 * gradients): the same packing and rank-ordered fold as
 * or_reduce_scatter_direct, with fp32 sources (no cast needed). */
void or_reduce_scatter_f32(const int64_t* d0, const int64_t* cols, int32_t n, int32_t N,
                           const float* src, int32_t op, float* red) {
    int64_t c[n > 0 ? n : 1], s[n > 0 ? n : 1], off[n > 0 ? n : 1],
        u[n > 0 ? n : 1], sz[3];
    or_plan(d0, cols, n, N, c, s, off, u, sz);
    int64_t S = sz[0], A = sz[2];
    for (int32_t j = 0; j < N; ++j) {
        for (int32_t i = 0; i < n; ++i) {
            int64_t v = or_valid_rows(d0[i], N, j);
#pragma omp parallel for schedule(static)
            for (int64_t row = 0; row < c[i]; ++row) {
                for (int64_t col = 0; col < cols[i]; ++col) {
                    int64_t dst = (int64_t)j * S + off[i] + row * cols[i] + col;
                    if (row >= v) {
                        red[dst] = 0.0f;
                        continue;
                    }
                    int64_t k = u[i] + ((int64_t)j * c[i] + row) * cols[i] + col;
                    float acc = src[k];
                    for (int32_t r = 1; r < N; ++r) acc = acc + src[(int64_t)r * A + k];
                    if (op == OR_AVG) acc = acc / (float)N;
                    red[dst] = acc;
                }
            }
        }
    }
    if (op == OR_SUM_THEN_DIV) {
        int64_t total = (int64_t)N * S;
#pragma omp parallel for schedule(static)
        for (int64_t k = 0; k < total; ++k) red[k] = red[k] / (float)N;
    }
}

/* ------------------------------------------------------------------ */
/* FP8 all-gather copy-in ("PyTorch FSDP2 Guide: Distributed LLM        */
/* Training with DTensor", Deep Dive "2. Native FP8 Training with       */
/* Float8Tensor": parameters in FP8 E4M3, the all-gather moves raw FP8  */
/* bytes).  The pages leave scaling open; reading: per-parameter        */
/* tensorwise dynamic scaling,                                          */
/*   amax_i  = max |x| over the whole parameter (all ranks),            */
/*   scale_i = 448 / max(amax_i, 1e-12)            (binary32),          */
/*   q       = e4m3_rn(clamp(x * scale_i, -448, 448)), pads 0x00.       */
/* E4M3 here is the "fn" encoding: bias 7, 3 mantissa bits, no          */
/* infinities, S.1111.111 is NaN, largest finite 448.                   */
/* ------------------------------------------------------------------ */

/* Round a finite |x| <= 448 (or NaN) to E4M3, nearest even, from the
 * format's definition. */
uint8_t or_e4m3_bits(float x) {
    if (x != x) return 0x7F; /* NaN */
    uint8_t sign = (f32_bits(x) >> 31) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a < 0.015625) { /* below 2^-6: subnormal grid of 2^-9 */
        double q = nearbyint(a * 512.0); /* 0..8; 8 is the smallest normal */
        return (uint8_t)(sign | (uint8_t)q);
    }
    int e = 0;
    double m = frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
    m *= 2.0;
    e -= 1; /* a = m * 2^e, m in [1, 2) */
    double r = nearbyint((m - 1.0) * 8.0);
    if (r == 8.0) {
        r = 0.0;
        e += 1;
    }
    int field = e + 7; /* 1..15 for 2^-6 <= a <= 448 */
    return (uint8_t)(sign | (uint8_t)(field << 3) | (uint8_t)r);
}

float or_fp8_scale(float amax) {
    float a = amax > 1e-12f ? amax : 1e-12f;
    return 448.0f / a;
}

float or_fp8_quant_input(float x, float scale) {
    float y = x * scale;
    if (y > 448.0f) y = 448.0f;
    if (y < -448.0f) y = -448.0f;
    return y;
}

void or_cast_e4m3(const float* x, uint8_t* y, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k) y[k] = or_e4m3_bits(x[k]);
}

/* scales[i] = 448 / max(amax_i, 1e-12), amax over parameter i's real rows */
void or_fp8_scales(const int64_t* d0, const int64_t* cols, int32_t n, int32_t N,
                   const float* master, float* scales) {
    int64_t c[n > 0 ? n : 1], s[n > 0 ? n : 1], off[n > 0 ? n : 1],
        u[n > 0 ? n : 1], sz[3];
    or_plan(d0, cols, n, N, c, s, off, u, sz);
    int64_t S = sz[0];
    for (int32_t i = 0; i < n; ++i) {
        float amax = 0.0f;
        for (int32_t r = 0; r < N; ++r) {
            int64_t v = or_valid_rows(d0[i], N, r);
            for (int64_t k = 0; k < v * cols[i]; ++k) {
                float a = fabsf(master[(int64_t)r * S + off[i] + k]);
                if (a > amax) amax = a;
            }
        }
        scales[i] = or_fp8_scale(amax);
    }
}

void or_copy_in_fp8(const int64_t* d0, const int64_t* cols, int32_t n, int32_t N,
                    const float* master, const float* scales, uint8_t* ag8) {
    int64_t c[n > 0 ? n : 1], s[n > 0 ? n : 1], off[n > 0 ? n : 1],
        u[n > 0 ? n : 1], sz[3];
    or_plan(d0, cols, n, N, c, s, off, u, sz);
    int64_t S = sz[0];
#pragma omp parallel for schedule(static)
    for (int32_t r = 0; r < N; ++r) {
        for (int32_t i = 0; i < n; ++i) {
            int64_t v = or_valid_rows(d0[i], N, r);
            for (int64_t row = 0; row < c[i]; ++row) {
                for (int64_t col = 0; col < cols[i]; ++col) {
                    int64_t k = (int64_t)r * S + off[i] + row * cols[i] + col;
                    ag8[k] = (row < v) ? or_e4m3_bits(or_fp8_quant_input(master[k], scales[i]))
                                       : (uint8_t)0;
                }
            }
        }
    }
}

void or_copy_out_fp8(const int64_t* d0, const int64_t* cols, int32_t n, int32_t N,
                     const uint8_t* ag8, uint8_t* arena8) {
    int64_t c[n > 0 ? n : 1], s[n > 0 ? n : 1], off[n > 0 ? n : 1],
        u[n > 0 ? n : 1], sz[3];
    or_plan(d0, cols, n, N, c, s, off, u, sz);
    int64_t S = sz[0];
    for (int32_t i = 0; i < n; ++i) {
#pragma omp parallel for schedule(static)
        for (int64_t row = 0; row < d0[i]; ++row) {
            int64_t r = row / c[i];
            int64_t local = row - r * c[i];
            for (int64_t col = 0; col < cols[i]; ++col)
                arena8[u[i] + row * cols[i] + col] = ag8[r * S + off[i] + local * cols[i] + col];
        }
    }
}

/* ------------------------------------------------------------------ */
/* a5 AdamW (decoupled weight decay), binary64, one rounding per store */
/* [ML] Fence 4 (AdamW built after sharding steps each shard);          */
/* [MS] "Working Principle" (update state uses gradient slices).       */
/* ------------------------------------------------------------------ */
void or_adamw(float* p, float* m, float* v, const float* g, int64_t count,
              double lr, double beta1, double beta2, double eps, double wd,
              int64_t step) {
    double bc1 = 1.0 - pow(beta1, (double)step);
    double bc2 = 1.0 - pow(beta2, (double)step);
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < count; ++k) {
        double pk = (double)p[k];
        double gk = (double)g[k];
        double mk = (double)m[k];
        double vk = (double)v[k];
        pk = pk * (1.0 - lr * wd);
        mk = beta1 * mk + (1.0 - beta1) * gk;
        vk = beta2 * vk + (1.0 - beta2) * gk * gk;
        double mhat = mk / bc1;
        double vhat = vk / bc2;
        pk = pk - lr * mhat / (sqrt(vhat) + eps);
        p[k] = (float)pk;
        m[k] = (float)mk;
        v[k] = (float)vk;
    }
}
