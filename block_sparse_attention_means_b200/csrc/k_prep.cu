// Input check, QRKC metric, row norms, strided K-means initialisation and
// per-iteration centroid operands.
#include "kernels.h"

namespace park {

// ---------------------------------------------------------------- input check
// One pass over the tensor with 16-byte loads: every element must be 0 or a
// finite value with 2^-40 <= |x| < 2^40 (the library's range precondition).
// For bf16, wide[h] (when given) is set for every head h holding an element
// with |x| >= 2^16 (none in unit-scale data): the centroid update of such a
// head takes its general 128-bit path instead of the float64 partial sums
// (k_sort.cu); and tiny_rows[r] (when given) for every row r holding a nonzero
// element with |x| < 2^-20 (about one row in ten thousand in unit-scale data),
// which the float64 partial sums cannot take exactly either.  With xnorm given
// (bf16 rows of 128 elements: 16 pieces, one per lane of a half warp) it also
// writes every row's ||x|| for the certified assign bound (float64 sum of
// squares, square root rounded up to float), so the K-means needs no second pass
// over X.
template <int BYTES>
__global__ void k_input_check(const uint4* __restrict__ x, size_t n16, int32_t* status, size_t per_head16,
                              int32_t* __restrict__ wide, uint8_t* __restrict__ tiny_rows, size_t row16,
                              float* __restrict__ xnorm) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;  // a multiple of 32
    const int lane = threadIdx.x & 31;
    bool bad = false;
    // warp-uniform trip count: the half-warp reductions below need every lane
    for (size_t i0 = (size_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31u); i0 < n16; i0 += stride) {
        const size_t i = i0 + lane;
        const bool in = i < n16;
        uint4 v = in ? x[i] : make_uint4(0u, 0u, 0u, 0u);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
        if (BYTES == 2 && xnorm != nullptr) {
            double ss = 0.0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const double lo = (double)__uint_as_float(w[q] << 16), hi = (double)__uint_as_float(w[q] & 0xffff0000u);
                ss = fma(lo, lo, ss);
                ss = fma(hi, hi, ss);
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (in && (lane & 15) == 0) xnorm[i >> 4] = round_up_f(__double2float_ru(sqrt(ss)));
        }
        bool narrow = true, tiny = false;
        if (BYTES == 2) {
            // both bf16 halves of a word at once: with x the two 15-bit magnitudes, x + c
            // sets bit 15 of a half exactly when its magnitude is >= 0x8000 - c (no carry
            // reaches the other half): nonzero (>= 1), exponent >= 87 (0x2B80), >= 167
            // (0x5380: beyond the range, or inf / NaN), >= 143 (0x4780: |x| >= 2^16) and
            // >= 107 (0x3580: |x| >= 2^-20)
            uint32_t a_bad = 0, a_wide = 0, a_tiny = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t x = w[q] & 0x7FFF7FFFu;
                const uint32_t nz = x + 0x7FFF7FFFu;
                a_bad |= nz & (~(x + 0x54805480u) | (x + 0x2C802C80u));
                a_wide |= x + 0x38803880u;
                a_tiny |= nz & ~(x + 0x4A804A80u);
            }
            bad |= (a_bad & 0x80008000u) != 0u;
            narrow = (a_wide & 0x80008000u) == 0u;
            tiny = (a_tiny & 0x80008000u) != 0u;
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t mag = w[q] & 0x7FFFFFFFu;
                int e = (w[q] >> 23) & 0xFF;
                bad |= !in_range_exp(e, mag);
            }
        }
        if (in && BYTES == 2 && !narrow && wide) atomicOr(wide + i / per_head16, 1);  // rare
        if (in && BYTES == 2 && tiny && tiny_rows) tiny_rows[i / row16] = 1;            // rare
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) set_status(status, PARK_ERR_RANGE);
}

int launch_input_check(const void* x, size_t n_elems, int dtype, int32_t* status, int32_t* wide,
                       size_t per_head_elems, uint8_t* tiny_rows, size_t row_elems, float* xnorm,
                       cudaStream_t st) {
    int eb = dtype == PARK_BF16 ? 2 : 4;
    size_t n16 = n_elems * eb / 16;
    int blocks = (int)((n16 + 255) / 256);
    ::park::prof_begin(st);
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    const size_t ph16 = per_head_elems * eb / 16;  // a head is a whole number of 16-byte pieces (D % 8 == 0)
    const size_t r16 = row_elems * eb / 16;          // and so is a row
    if (eb == 2)
        k_input_check<2><<<blocks, 256, 0, st>>>((const uint4*)x, n16, status, ph16 ? ph16 : 1, wide,
                                                 r16 ? tiny_rows : nullptr, r16 ? r16 : 1,
                                                 r16 == 16 ? xnorm : nullptr);
    else
        k_input_check<4><<<blocks, 256, 0, st>>>((const uint4*)x, n16, status, ph16 ? ph16 : 1, nullptr, nullptr, 1,
                                                 nullptr);
    PARK_TRY_LAUNCH("k_input_check", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- metric
// M = (1/N) sum_i q_i q_i^T in float64, exploiting symmetry.  Pass 1: one CTA
// per (row chunk, head) sums the outer products of its rows into the upper
// triangle of 8 x 8 blocks (136 blocks for D = 128); thread i owns rows
// 8 ta + 4 (i & 1) + 0..3 and columns 8 tb + 0..7 of block i >> 1 (ta <= tb),
// reading the rows from shared memory with 16-byte loads.  Pass 2 adds the
// chunk partials in chunk order, divides by N and writes M[a][b] = M[b][a], so
// M is exactly symmetric.
constexpr int kMetricRB = 32;  // rows staged per step

template <typename T>
__global__ __launch_bounds__(272) void k_metric_partial(const T* __restrict__ Q, int N, int D, int rows_per_chunk,
                                                        double* __restrict__ part) {
    __shared__ __align__(16) double qs[kMetricRB][128];
    const int bh = blockIdx.y, c = blockIdx.x, nch = gridDim.x;
    const T* X = Q + (size_t)bh * N * D;
    const int r0 = c * rows_per_chunk, r1 = min(N, r0 + rows_per_chunk);
    const int t = threadIdx.x, bi = t >> 1, hf = t & 1;
    int tb = (int)((sqrt(8.0 * bi + 1.0) - 1.0) * 0.5);
    while ((tb + 1) * (tb + 2) / 2 <= bi) ++tb;
    while (tb * (tb + 1) / 2 > bi) --tb;
    const int ta = bi - tb * (tb + 1) / 2;
    const int a0 = 8 * ta + 4 * hf, b0 = 8 * tb;
    const bool active = b0 < D;  // D is a multiple of 32
    double acc[4][8];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[u][v] = 0.0;
    // the next block of rows is fetched into registers while the current one is used
    constexpr int PER = (kMetricRB * 128 + 271) / 272;
    float pre[PER];  // inputs are exact in float32
    auto fetch = [&](int base) {
#pragma unroll
        for (int v = 0; v < PER; ++v) {
            const int e = t + 272 * v, rr = e >> 7, jj = e & 127;
            pre[v] = (e < kMetricRB * 128 && base + rr < r1 && jj < D)
                         ? Elem<T>::to_float(X + (size_t)(base + rr) * D, jj) : 0.f;
        }
    };
    if (r0 < r1) fetch(r0);
    for (int base = r0; base < r1; base += kMetricRB) {
        const int nr = min(kMetricRB, r1 - base);
        __syncthreads();
#pragma unroll
        for (int v = 0; v < PER; ++v) {
            const int e = t + 272 * v;
            if (e < kMetricRB * 128) qs[e >> 7][e & 127] = (double)pre[v];
        }
        __syncthreads();
        if (base + kMetricRB < r1) fetch(base + kMetricRB);
        if (active) {
            for (int rr = 0; rr < nr; ++rr) {
                double qa[4], qb[8];
#pragma unroll
                for (int u = 0; u < 4; u += 2) {
                    const double2 x = *reinterpret_cast<const double2*>(&qs[rr][a0 + u]);
                    qa[u] = x.x;
                    qa[u + 1] = x.y;
                }
#pragma unroll
                for (int v = 0; v < 8; v += 2) {
                    const double2 x = *reinterpret_cast<const double2*>(&qs[rr][b0 + v]);
                    qb[v] = x.x;
                    qb[v + 1] = x.y;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc[u][v] = __fma_rn(qa[u], qb[v], acc[u][v]);
            }
        }
    }
    if (!active) return;
    double* P = part + ((size_t)bh * nch + c) * D * D;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) P[(a0 + u) * D + b0 + v] = acc[u][v];
}

// D = 128: the same partials on the float64 tensor cores (mma.sync m8n8k4 f64,
// exact products and float64 accumulation).  256 threads; warp w owns the block
// rows w and 15 - w of the upper triangle of 8 x 8 blocks (17 blocks, the B
// fragments of row 15 - w are those of row w's last w + 1 blocks).  Rows are
// staged 32 at a time in shared memory as float64 (row pitch 136 doubles: the
// four rows of a fragment load fall in different bank halves); k-steps of 4
// rows.  Fragment layouts (PTX ISA, m8n8k4 .f64): A[r][k] and B[k][c] are held
// by lane 4 r + k and 4 c + k, D[r][2 (l % 4) + {0, 1}] by lane l = 4 r + ...
constexpr int kMetricPitch = 136;

__device__ __forceinline__ void dmma_m8n8k4(double& d0, double& d1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(d0), "+d"(d1)
                 : "d"(a), "d"(b));
}

// Warp W's part: rows W and 15 - W (compile-time, so that every accumulator
// index is static).
template <int W>
__device__ __forceinline__ void metric_mma_rows(const double* __restrict__ qs, int nk, double (&acc)[17][2],
                                                int lane) {
    constexpr int ta0 = W, ta1 = 15 - W;
    const int fr = lane >> 2, fk = lane & 3;
#pragma unroll 2
    for (int k0 = 0; k0 < nk; k0 += 4) {
        const double* rowp = qs + (k0 + fk) * kMetricPitch + fr;
        const double a0 = rowp[8 * ta0], a1 = rowp[8 * ta1];
#pragma unroll
        for (int q = 0; q < 16 - W; ++q) {  // blocks (ta0, ta0 + q); (ta1, ta0 + q) when ta0 + q >= ta1
            const double b = rowp[8 * (ta0 + q)];
            dmma_m8n8k4(acc[q][0], acc[q][1], a0, b);
            if (ta0 + q >= ta1) dmma_m8n8k4(acc[16 - W + (ta0 + q - ta1)][0], acc[16 - W + (ta0 + q - ta1)][1], a1, b);
        }
    }
}

template <int W>
__device__ __forceinline__ void metric_mma_store(double* __restrict__ P, const double (&acc)[17][2], int lane) {
    constexpr int D = 128, ta0 = W, ta1 = 15 - W;
    const int cr = lane >> 2, cc = 2 * (lane & 3);
#pragma unroll
    for (int q = 0; q < 16 - W; ++q) {
        const int tb = ta0 + q;
        P[(8 * ta0 + cr) * D + 8 * tb + cc] = acc[q][0];
        P[(8 * ta0 + cr) * D + 8 * tb + cc + 1] = acc[q][1];
        if (tb >= ta1) {
            P[(8 * ta1 + cr) * D + 8 * tb + cc] = acc[16 - W + (tb - ta1)][0];
            P[(8 * ta1 + cr) * D + 8 * tb + cc + 1] = acc[16 - W + (tb - ta1)][1];
        }
    }
}

template <typename T>
__global__ __launch_bounds__(256) void k_metric_partial_mma(const T* __restrict__ Q, int N, int rows_per_chunk,
                                                            double* __restrict__ part) {
    constexpr int D = 128, RB = 32;
    __shared__ __align__(16) double qs[RB * kMetricPitch];
    const int bh = blockIdx.y, c = blockIdx.x, nch = gridDim.x;
    const T* X = Q + (size_t)bh * N * D;
    const int r0 = c * rows_per_chunk, r1 = min(N, r0 + rows_per_chunk);
    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    double acc[17][2];
#pragma unroll
    for (int b = 0; b < 17; ++b) acc[b][0] = acc[b][1] = 0.0;
    constexpr int PER = RB * D / 256;  // 16 elements per thread per block of rows
    float pre[PER];                    // inputs are exact in float32
    auto fetch = [&](int base) {
#pragma unroll
        for (int v = 0; v < PER; ++v) {
            const int e = t + 256 * v, rr = e >> 7, jj = e & 127;
            pre[v] = base + rr < r1 ? Elem<T>::to_float(X + (size_t)(base + rr) * D, jj) : 0.f;
        }
    };
    if (r0 < r1) fetch(r0);
    for (int base = r0; base < r1; base += RB) {
        __syncthreads();
#pragma unroll
        for (int v = 0; v < PER; ++v) {
            const int e = t + 256 * v;
            qs[(e >> 7) * kMetricPitch + (e & 127)] = (double)pre[v];  // rows past the end are 0
        }
        __syncthreads();
        if (base + RB < r1) fetch(base + RB);
        switch (w) {  // warp-uniform
            case 0: metric_mma_rows<0>(qs, RB, acc, lane); break;
            case 1: metric_mma_rows<1>(qs, RB, acc, lane); break;
            case 2: metric_mma_rows<2>(qs, RB, acc, lane); break;
            case 3: metric_mma_rows<3>(qs, RB, acc, lane); break;
            case 4: metric_mma_rows<4>(qs, RB, acc, lane); break;
            case 5: metric_mma_rows<5>(qs, RB, acc, lane); break;
            case 6: metric_mma_rows<6>(qs, RB, acc, lane); break;
            default: metric_mma_rows<7>(qs, RB, acc, lane); break;
        }
    }
    double* P = part + ((size_t)bh * nch + c) * D * D;
    switch (w) {
        case 0: metric_mma_store<0>(P, acc, lane); break;
        case 1: metric_mma_store<1>(P, acc, lane); break;
        case 2: metric_mma_store<2>(P, acc, lane); break;
        case 3: metric_mma_store<3>(P, acc, lane); break;
        case 4: metric_mma_store<4>(P, acc, lane); break;
        case 5: metric_mma_store<5>(P, acc, lane); break;
        case 6: metric_mma_store<6>(P, acc, lane); break;
        default: metric_mma_store<7>(P, acc, lane); break;
    }
}

__global__ void k_metric_reduce(const double* __restrict__ part, int nch, int N, int D, double* __restrict__ M,
                                double* __restrict__ M_out) {
    const int bh = blockIdx.y;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= D * D) return;
    const int a = e / D, b = e - a * D;
    // entry (a, b) of the upper triangle of 8 x 8 blocks that holds {a, b}
    const int ua = (a >> 3) <= (b >> 3) ? a : b, ub = (a >> 3) <= (b >> 3) ? b : a;
    const int src = ua * D + ub;
    double s = 0.0;
    for (int c = 0; c < nch; ++c) s += part[((size_t)bh * nch + c) * D * D + src];
    const double m = s / (double)N;
    M[(size_t)bh * D * D + e] = m;
    if (M_out) M_out[(size_t)bh * D * D + e] = m;
}

int launch_metric(const void* Q, int dtype, int BH, int N, int D, double* part, int nchunks, double* M,
                  double* M_out, cudaStream_t st) {
    if (D > 128 || D % 32 != 0) return PARK_ERR_UNSUPPORTED;
    int rpc = (N + nchunks - 1) / nchunks;
    dim3 g1(nchunks, BH);
    ::park::prof_begin(st);
    if (dtype == PARK_BF16 && D == 128)
        k_metric_partial_mma<bf16_t><<<g1, 256, 0, st>>>((const bf16_t*)Q, N, rpc, part);
    else if (D == 128)
        k_metric_partial_mma<float><<<g1, 256, 0, st>>>((const float*)Q, N, rpc, part);
    else if (dtype == PARK_BF16)
        k_metric_partial<bf16_t><<<g1, 272, 0, st>>>((const bf16_t*)Q, N, D, rpc, part);
    else
        k_metric_partial<float><<<g1, 272, 0, st>>>((const float*)Q, N, D, rpc, part);
    PARK_TRY_LAUNCH("k_metric_partial", st);
    dim3 g2((D * D + 255) / 256, BH);
    ::park::prof_begin(st);
    k_metric_reduce<<<g2, 256, 0, st>>>(part, nchunks, N, D, M, M_out);
    PARK_TRY_LAUNCH("k_metric_reduce", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- strided init
// c_k = x_floor(k N / K) (pages silent on initialisation; deterministic choice).
__global__ void k_strided_init(const uint8_t* __restrict__ X, int N, int K, int row_bytes, uint8_t* __restrict__ C) {
    int k = blockIdx.x, bh = blockIdx.y;
    long long src = ((long long)k * N) / K;
    const uint8_t* s = X + ((size_t)bh * N + src) * row_bytes;
    uint8_t* d = C + ((size_t)bh * K + k) * row_bytes;
    for (int b = threadIdx.x * 4; b < row_bytes; b += blockDim.x * 4)
        *(uint32_t*)(d + b) = *(const uint32_t*)(s + b);
}

int launch_strided_init(const void* X, int dtype, int BH, int N, int D, int K, void* C, cudaStream_t st) {
    int rb = D * (dtype == PARK_BF16 ? 2 : 4);
    ::park::prof_begin(st);
    k_strided_init<<<dim3(K, BH), 64, 0, st>>>((const uint8_t*)X, N, K, rb, (uint8_t*)C);
    PARK_TRY_LAUNCH("k_strided_init", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- centroid operands
// Euclidean operands, per centroid: bias = ||c||^2 and the per-head maxima
// ||c|| and |bias| used by the certified bound (the score GEMM reads the
// centroids themselves, w = c).  One CTA of D threads per (centroid, head);
// float64 sums in a fixed tree.
template <typename T>
__global__ void k_centroid_prep(const T* __restrict__ C, int K, int D, float* __restrict__ bias32, int bias_ld,
                                double* __restrict__ bias64, float* __restrict__ wmax, float* __restrict__ bmax) {
    __shared__ double red[128];
    int k = blockIdx.x, bh = blockIdx.y, a = threadIdx.x;
    const T* c = C + ((size_t)bh * K + k) * D;
    const double ca = Elem<T>::to_double(c, a);
    red[a] = ca * ca;
    __syncthreads();
    for (int s = 64; s > 0; s >>= 1) {
        if (a < s && a + s < D) red[a] += red[a + s];
        __syncthreads();
    }
    if (k == 0)  // columns past K read +inf, so a score GEMM over whole 128-column chunks never picks them
        for (int j = K + a; j < ((K + 127) & ~127); j += blockDim.x)
            bias32[(size_t)bh * bias_ld + j] = __int_as_float(0x7f800000);
    if (a == 0) {
        const double b = red[0];
        bias64[(size_t)bh * K + k] = b;
        bias32[(size_t)bh * bias_ld + k] = __double2float_rn(b);
        atomic_max_nonneg(wmax + bh, round_up_f(__double2float_ru(sqrt(b))));
        atomic_max_nonneg(bmax + bh, round_up_f(__double2float_ru(fabs(b))));
    }
}

// QRKC operands for 64 centroids per CTA: M (symmetric, float64) and the
// centroids (transposed: Cs[b][c]) are staged once in shared memory; thread t
// owns columns 4 (t % 32) .. + 3 and centroids 8 (t / 32) .. + 7 and forms
// w_a = sum_b M[b][a] c_b for them, summing over b in order (four M values and
// eight centroid values per step: 32 FMAs per 6 shared loads).  A warp holds whole
// rows w of its eight centroids, so bias = c . w and ||w||^2 are reduced within
// the warp in a fixed order.
// w and the bias are taken for 2^-e M, e the binary exponent of the head's
// largest diagonal entry (|M_ab| <= max_a M_aa), so that the float32 scores stay
// far from overflow over the whole input range (|x| < 2^40 gives M up to 2^80).
// A power-of-two scale is exact in float64 and multiplies every score of the
// head by the same factor, so it changes no argmin.
constexpr int kPrepCents = 64;

template <typename T>
__global__ __launch_bounds__(256) void k_centroid_prep_metric(const T* __restrict__ C, int K, int D,
                                                              const double* __restrict__ Mall,
                                                              uint16_t* __restrict__ wop, float* __restrict__ bias32,
                                                              int bias_ld, double* __restrict__ bias64,
                                                              double* __restrict__ w64, float* __restrict__ wmax,
                                                              float* __restrict__ bmax) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    double* Ms = reinterpret_cast<double*>(smem_raw);  // [D][D]
    double* Cs = Ms + D * D;                          // [D][kPrepCents]: Cs[b][c]
    __shared__ double s_scale;
    const int bh = blockIdx.y, k0 = blockIdx.x * kPrepCents, t = threadIdx.x;
    const int lane = t & 31, cb = t >> 5;  // column block (4 columns), centroid block (8 centroids)
    const int a0 = 4 * lane, c0 = 8 * cb;
    const double2* M2 = reinterpret_cast<const double2*>(Mall + (size_t)bh * D * D);
    double2* Ms2 = reinterpret_cast<double2*>(Ms);
    const int n2 = D * D / 2;
    for (int i0 = t; i0 < n2; i0 += 256 * 8) {  // eight 16-byte loads in flight per thread
        double2 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (i0 + 256 * u < n2) v[u] = M2[i0 + 256 * u];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (i0 + 256 * u < n2) Ms2[i0 + 256 * u] = v[u];
    }
    for (int i = t; i < kPrepCents * D; i += blockDim.x) {
        const int c = i / D, j = i - c * D, k = k0 + c;
        Cs[j * kPrepCents + c] = k < K ? Elem<T>::to_double(C + ((size_t)bh * K + k) * D, j) : 0.0;
    }
    if (blockIdx.x == 0)  // columns past K read +inf, so a score GEMM over whole 128-column chunks never picks them
        for (int j = K + t; j < ((K + 127) & ~127); j += blockDim.x)
            bias32[(size_t)bh * bias_ld + j] = __int_as_float(0x7f800000);
    __syncthreads();
    if (t < 32) {
        double dm = 0.0;
        for (int j = t; j < D; j += 32) dm = fmax(dm, Ms[j * D + j]);
        dm = warp_max(dm);
        if (t == 0) s_scale = dm > 0.0 ? ldexp(1.0, -ilogb(dm)) : 1.0;
    }
    __syncthreads();
    const double scale = s_scale;
    const bool act = a0 < D;  // D is a multiple of 32: a thread's four columns are all in or all out
    double w[8][4];
#pragma unroll
    for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) w[c][j] = 0.0;
    if (act) {
        for (int b = 0; b < D; ++b) {
            const double2 m01 = *reinterpret_cast<const double2*>(Ms + b * D + a0);
            const double2 m23 = *reinterpret_cast<const double2*>(Ms + b * D + a0 + 2);
            const double mv[4] = {m01.x, m01.y, m23.x, m23.y};
#pragma unroll
            for (int c2 = 0; c2 < 4; ++c2) {
                const double2 cv = *reinterpret_cast<const double2*>(Cs + b * kPrepCents + c0 + 2 * c2);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    w[2 * c2][j] = __fma_rn(mv[j], cv.x, w[2 * c2][j]);
                    w[2 * c2 + 1][j] = __fma_rn(mv[j], cv.y, w[2 * c2 + 1][j]);
                }
            }
        }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const int k = k0 + c0 + c;
        double pb = 0.0, pn = 0.0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            w[c][j] *= scale;  // exact
            if (act) {
                pb = __fma_rn(Cs[(a0 + j) * kPrepCents + c0 + c], w[c][j], pb);
                pn = __fma_rn(w[c][j], w[c][j], pn);
            }
        }
        if (act && k < K) {
            double* wd = w64 + ((size_t)bh * K + k) * D + a0;
            reinterpret_cast<double2*>(wd)[0] = make_double2(w[c][0], w[c][1]);
            reinterpret_cast<double2*>(wd)[1] = make_double2(w[c][2], w[c][3]);
            if (wop != nullptr) {
                uint32_t hi2[2], lo2[2];
#pragma unroll
                for (int j = 0; j < 4; j += 2) {
                    uint16_t h[2], l[2];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        h[q] = double_to_bf16_bits(w[c][j + q]);
                        const double hid = (double)__uint_as_float(((uint32_t)h[q]) << 16);
                        l[q] = double_to_bf16_bits(w[c][j + q] - hid);  // w - hi is exact
                    }
                    hi2[j >> 1] = (uint32_t)h[0] | ((uint32_t)h[1] << 16);
                    lo2[j >> 1] = (uint32_t)l[0] | ((uint32_t)l[1] << 16);
                }
                uint16_t* row = wop + ((size_t)bh * K + k) * (2 * D);
                *reinterpret_cast<uint2*>(row + a0) = make_uint2(hi2[0], hi2[1]);
                *reinterpret_cast<uint2*>(row + D + a0) = make_uint2(lo2[0], lo2[1]);
            }
        }
        pb = warp_sum(pb);
        pn = warp_sum(pn);
        if (lane == 0 && k < K) {
            bias64[(size_t)bh * K + k] = pb;
            bias32[(size_t)bh * bias_ld + k] = __double2float_rn(pb);
            atomic_max_nonneg(wmax + bh, round_up_f(__double2float_ru(sqrt(pn))));
            atomic_max_nonneg(bmax + bh, round_up_f(__double2float_ru(fabs(pb))));
        }
    }
}

int launch_centroid_prep(const void* C, int dtype, int BH, int K, int D, const double* M, CentroidOps ops,
                         cudaStream_t st) {
    if (D > 128) return PARK_ERR_UNSUPPORTED;  // one thread per coordinate
    dim3 g(K, BH);
    bool metric = M != nullptr;
    if (metric) {  // tiled form: M staged once per 16 centroids
        const dim3 gm((K + kPrepCents - 1) / kPrepCents, BH);
        const size_t sm = (size_t)D * D * 8 + (size_t)kPrepCents * D * 8;
        ::park::prof_begin(st);
        if (dtype == PARK_BF16) {
            cudaFuncSetAttribute(k_centroid_prep_metric<bf16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            k_centroid_prep_metric<bf16_t><<<gm, 256, sm, st>>>((const bf16_t*)C, K, D, M, (uint16_t*)ops.w,
                                                               ops.bias32, ops.bias_ld, ops.bias64, ops.w64,
                                                               ops.wmax, ops.bmax);
        } else {
            cudaFuncSetAttribute(k_centroid_prep_metric<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            k_centroid_prep_metric<float><<<gm, 256, sm, st>>>((const float*)C, K, D, M, (uint16_t*)ops.w, ops.bias32,
                                                              ops.bias_ld, ops.bias64, ops.w64, ops.wmax, ops.bmax);
        }
        PARK_TRY_LAUNCH("k_centroid_prep_metric", st);
        return PARK_OK;
    }
    ::park::prof_begin(st);
    if (dtype == PARK_BF16)
        k_centroid_prep<bf16_t><<<g, D, 0, st>>>((const bf16_t*)C, K, D, ops.bias32, ops.bias_ld, ops.bias64, ops.wmax,
                                                 ops.bmax);
    else
        k_centroid_prep<float><<<g, D, 0, st>>>((const float*)C, K, D, ops.bias32, ops.bias_ld, ops.bias64, ops.wmax,
                                                ops.bmax);
    PARK_TRY_LAUNCH("k_centroid_prep", st);
    return PARK_OK;
}

}  // namespace park
