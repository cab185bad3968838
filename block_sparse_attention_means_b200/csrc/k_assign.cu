// K-means assign step: a(i) = argmin_k D(x_i, c_k), ties to the lowest k.
//
// Fast path (bf16 inputs, k_assign_tc.cu): one tensor-core GEMM gives float scores
//   s~_k = bias_k - 2 x . w_k      (Euclidean: w = c, bias = ||c||^2;
//                                  QRKC: w = M c as bf16 hi+lo, bias = c^T M c)
// which equal D(x, c_k) - x^T M x up to a rigorous per-row error bound beta.
// The epilogue keeps the smallest and second smallest score per row.  The
// winner is certified when the runner-up is more than 2 beta above it;
// otherwise the row is listed for a float64 rescore against every centroid
// (k_rescore_full), so labels agree with a float64 evaluation of the definition.
#include <algorithm>

#include "kernels.h"

namespace park {


// ---------------------------------------------------------------- float64 rescore
// Every row of every head against every centroid, one warp per row (the float32
// input path, which has no tensor-core filter).  Euclidean distance:
// sum_j (x_j - c_j)^2.  QRKC: c^T M c - 2 x . (M c), the distance minus the row
// constant x^T M x.  Ties go to the lowest index.
// Rows row0 .. N-1 of every head (row0 = 0: all rows).
template <typename T, bool METRIC>
__global__ void k_recheck(const T* __restrict__ X, const T* __restrict__ C, const double* __restrict__ w64,
                          const double* __restrict__ b64, int N, int D, int K, int32_t* __restrict__ labels,
                          int BH, int row0) {
    const int lane = threadIdx.x & 31;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    const int per_head = N - row0, total_rows = BH * per_head;
    for (int e = gw; e < total_rows; e += nw) {
        const int bh = e / per_head;
        const int gr = bh * N + row0 + (e - bh * per_head);
        const T* x = X + (size_t)gr * D;
        double xv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            int j = lane + 32 * u;
            xv[u] = j < D ? Elem<T>::to_double(x, j) : 0.0;
        }
        auto dist = [&](int k) -> double {
            double s = 0.0;
            if (METRIC) {
                const double* w = w64 + ((size_t)bh * K + k) * D;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    int j = lane + 32 * u;
                    if (j < D) s = __fma_rn(xv[u], w[j], s);
                }
                s = warp_sum(s);
                return b64[(size_t)bh * K + k] - 2.0 * s;
            } else {
                const T* c = C + ((size_t)bh * K + k) * D;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    int j = lane + 32 * u;
                    if (j < D) {
                        double d = xv[u] - Elem<T>::to_double(c, j);
                        s = __fma_rn(d, d, s);
                    }
                }
                return warp_sum(s);
            }
        };
        double bd = __longlong_as_double(0x7ff0000000000000ll);
        int best = 0;
        for (int k = 0; k < K; ++k) {
            double d = dist(k);
            if (d < bd) {
                bd = d;
                best = k;
            }
        }
        if (lane == 0) labels[gr] = best;
    }
}

// Full rescore of the rows the tensor-core assign could not certify, listed per
// head.  The listed rows are taken in groups of up to eight rows of one head;
// every CTA walks the groups of all heads (g = blockIdx.x, blockIdx.x +
// gridDim.x, ...), so heads with long lists do not hold up the launch.  A
// group's rows are staged in shared memory as float64, and thread t scores the
// centroids k0 + t and k0 + 256 + t (k0 = 0, 512, ...) against all of them: one
// thread per centroid, each distance a sequential float64 sum over the D
// elements, so no lanes have to be reduced per distance.  The smallest distance
// of a row, ties to the lowest index, is kept per thread (its centroids come in
// increasing order) and then found over the CTA.
constexpr int kRescoreRows = 8;
constexpr int kRescoreThreads = 256;

// elements j and j + 1 of a row as float64 (j even; rows are 16-byte aligned)
__device__ __forceinline__ double2 load2_f64(const double* p, int j) {
    return *reinterpret_cast<const double2*>(p + j);
}
__device__ __forceinline__ double2 load2_f64(const float* p, int j) {
    const float2 v = *reinterpret_cast<const float2*>(p + j);
    return make_double2((double)v.x, (double)v.y);
}
__device__ __forceinline__ double2 load2_f64(const bf16_t* p, int j) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p + j);
    return make_double2((double)__uint_as_float(w << 16), (double)__uint_as_float(w & 0xffff0000u));
}

template <typename T, bool METRIC>
__global__ __launch_bounds__(kRescoreThreads, 2) void k_rescore_full(
    const T* __restrict__ X, const T* __restrict__ C, const double* __restrict__ w64,
    const double* __restrict__ b64, int N, int D, int K, int BH, int32_t* __restrict__ labels,
    const int32_t* __restrict__ rows, const int32_t* __restrict__ counts, int64_t* __restrict__ counters,
    int cnt_slot) {
    constexpr int R = kRescoreRows;
    __shared__ __align__(16) double sx[R][128];
    __shared__ double s_best[kRescoreThreads / 32][R];
    __shared__ int s_idx[kRescoreThreads / 32][R];
    extern __shared__ int s_pref[];  // [BH + 1]: first group of each head
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    if (t == 0) {
        int a = 0;
        long long total = 0;
        for (int h = 0; h < BH; ++h) {
            s_pref[h] = a;
            a += (counts[h] + R - 1) / R;
            total += counts[h];
        }
        s_pref[BH] = a;
        if (blockIdx.x == 0 && counters != nullptr && total > 0) {
            atomicAdd((unsigned long long*)(counters + cnt_slot), (unsigned long long)total);
            atomicAdd((unsigned long long*)(counters + PARK_CNT_FULL_RESCORE), (unsigned long long)total);
        }
    }
    __syncthreads();
    const int G = s_pref[BH];
    for (int g = blockIdx.x; g < G; g += gridDim.x) {
        int bh = 0;
        while (s_pref[bh + 1] <= g) ++bh;
        const int g0 = (g - s_pref[bh]) * R;
        const int nr = min(R, counts[bh] - g0);
        const int32_t* list = rows + (size_t)bh * N + g0;
        for (int i = t; i < R * D; i += kRescoreThreads) {
            const int r = i / D, j = i - r * D;
            const int gr = list[r < nr ? r : 0];  // rows past the group repeat its first row
            sx[r][j] = Elem<T>::to_double(X + (size_t)gr * D, j);
        }
        __syncthreads();
        double bd[R];
        int best[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            bd[r] = __longlong_as_double(0x7ff0000000000000ll);
            best[r] = K;
        }
        for (int k0 = 0; k0 + t < K; k0 += 2 * kRescoreThreads) {
            const int ka = k0 + t, kb = ka + kRescoreThreads;
            const bool vb = kb < K;
            double acc_a[R], acc_b[R];
#pragma unroll
            for (int r = 0; r < R; ++r) acc_a[r] = acc_b[r] = 0.0;
            if (METRIC) {
                const double* pa = w64 + ((size_t)bh * K + ka) * D;
                const double* pb = w64 + ((size_t)bh * K + (vb ? kb : ka)) * D;
                for (int j = 0; j < D; j += 2) {
                    const double2 a2 = load2_f64(pa, j), b2 = load2_f64(pb, j);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const double2 x2 = *reinterpret_cast<const double2*>(&sx[r][j]);
                        acc_a[r] = __fma_rn(x2.x, a2.x, acc_a[r]);
                        acc_a[r] = __fma_rn(x2.y, a2.y, acc_a[r]);
                        acc_b[r] = __fma_rn(x2.x, b2.x, acc_b[r]);
                        acc_b[r] = __fma_rn(x2.y, b2.y, acc_b[r]);
                    }
                }
            } else {
                const T* pa = C + ((size_t)bh * K + ka) * D;
                const T* pb = C + ((size_t)bh * K + (vb ? kb : ka)) * D;
                for (int j = 0; j < D; j += 2) {
                    const double2 a2 = load2_f64(pa, j), b2 = load2_f64(pb, j);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const double2 x2 = *reinterpret_cast<const double2*>(&sx[r][j]);
                        double d = x2.x - a2.x;
                        acc_a[r] = __fma_rn(d, d, acc_a[r]);
                        d = x2.y - a2.y;
                        acc_a[r] = __fma_rn(d, d, acc_a[r]);
                        d = x2.x - b2.x;
                        acc_b[r] = __fma_rn(d, d, acc_b[r]);
                        d = x2.y - b2.y;
                        acc_b[r] = __fma_rn(d, d, acc_b[r]);
                    }
                }
            }
            const double ba = METRIC ? b64[(size_t)bh * K + ka] : 0.0;
            const double bb = METRIC && vb ? b64[(size_t)bh * K + kb] : 0.0;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const double da = METRIC ? ba - 2.0 * acc_a[r] : acc_a[r];
                if (da < bd[r]) {
                    bd[r] = da;
                    best[r] = ka;
                }
                const double db = METRIC ? bb - 2.0 * acc_b[r] : acc_b[r];
                if (vb && db < bd[r]) {
                    bd[r] = db;
                    best[r] = kb;
                }
            }
        }
        // smallest (distance, index) over the CTA
#pragma unroll
        for (int r = 0; r < R; ++r) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double od = __shfl_xor_sync(0xffffffffu, bd[r], off);
                const int oi = __shfl_xor_sync(0xffffffffu, best[r], off);
                if (od < bd[r] || (od == bd[r] && oi < best[r])) {
                    bd[r] = od;
                    best[r] = oi;
                }
            }
            if (lane == 0) {
                s_best[warp][r] = bd[r];
                s_idx[warp][r] = best[r];
            }
        }
        __syncthreads();
        if (t < nr) {
            double b = s_best[0][t];
            int bi = s_idx[0][t];
            for (int q = 1; q < kRescoreThreads / 32; ++q)
                if (s_best[q][t] < b || (s_best[q][t] == b && s_idx[q][t] < bi)) {
                    b = s_best[q][t];
                    bi = s_idx[q][t];
                }
            labels[list[t]] = bi;
        }
        __syncthreads();  // sx, s_best and s_idx are reused by the next group
    }
}

int launch_recheck_rows(const void* X, int dtype, int BH, int N, int D, int K, const void* C, const double* w64,
                        const double* b64, int32_t* labels, int row0, int num_sms, cudaStream_t st) {
    if (D > 128) return PARK_ERR_UNSUPPORTED;
    if (row0 >= N) return PARK_OK;
    const bool metric = w64 != nullptr;
    const int blocks = num_sms * 8;
    ::park::prof_begin(st);
    if (dtype == PARK_BF16) {
        if (metric)
            k_recheck<bf16_t, true><<<blocks, 256, 0, st>>>((const bf16_t*)X, (const bf16_t*)C, w64, b64, N, D, K,
                                                            labels, BH, row0);
        else
            k_recheck<bf16_t, false><<<blocks, 256, 0, st>>>((const bf16_t*)X, (const bf16_t*)C, w64, b64, N, D, K,
                                                             labels, BH, row0);
    } else {
        if (metric)
            k_recheck<float, true><<<blocks, 256, 0, st>>>((const float*)X, (const float*)C, w64, b64, N, D, K,
                                                           labels, BH, row0);
        else
            k_recheck<float, false><<<blocks, 256, 0, st>>>((const float*)X, (const float*)C, w64, b64, N, D, K,
                                                            labels, BH, row0);
    }
    PARK_TRY_LAUNCH("k_recheck", st);
    return PARK_OK;
}

int launch_recheck(const void* X, int dtype, int BH, int N, int D, int K, const void* C, const double* w64,
                   const double* b64, int32_t* labels, Lists lists, int all_rows, int num_sms,
                   int64_t* counters, int cnt_slot, cudaStream_t st) {
    if (D > 128) return PARK_ERR_UNSUPPORTED;
    const bool metric = w64 != nullptr;
    if (all_rows) return launch_recheck_rows(X, dtype, BH, N, D, K, C, w64, b64, labels, 0, num_sms, st);
    ::park::prof_begin(st);
    const int blocks = num_sms * 2;
    const size_t sm = (size_t)(BH + 1) * sizeof(int);
    if (dtype == PARK_BF16) {
        if (metric)
            k_rescore_full<bf16_t, true><<<blocks, kRescoreThreads, sm, st>>>(
                (const bf16_t*)X, (const bf16_t*)C, w64, b64, N, D, K, BH, labels, lists.full_row, lists.counts,
                counters, cnt_slot);
        else
            k_rescore_full<bf16_t, false><<<blocks, kRescoreThreads, sm, st>>>(
                (const bf16_t*)X, (const bf16_t*)C, w64, b64, N, D, K, BH, labels, lists.full_row, lists.counts,
                counters, cnt_slot);
    } else {
        if (metric)
            k_rescore_full<float, true><<<blocks, kRescoreThreads, sm, st>>>(
                (const float*)X, (const float*)C, w64, b64, N, D, K, BH, labels, lists.full_row, lists.counts,
                counters, cnt_slot);
        else
            k_rescore_full<float, false><<<blocks, kRescoreThreads, sm, st>>>(
                (const float*)X, (const float*)C, w64, b64, N, D, K, BH, labels, lists.full_row, lists.counts,
                counters, cnt_slot);
    }
    PARK_TRY_LAUNCH("k_rescore_full", st);
    return PARK_OK;
}

}  // namespace park
