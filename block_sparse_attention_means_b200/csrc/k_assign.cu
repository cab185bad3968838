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

// Full rescore (mode 1) with one CTA per listed row: warp w takes centroids
// w, w + 8, ..., two at a time; the CTA keeps the smallest distance, ties to the
// lowest index.
template <typename T, bool METRIC>
__global__ __launch_bounds__(256) void k_rescore_full(const T* __restrict__ X, const T* __restrict__ C,
                                                      const double* __restrict__ w64, const double* __restrict__ b64,
                                                      int N, int D, int K, int32_t* __restrict__ labels,
                                                      const int32_t* __restrict__ rows,
                                                      const int32_t* __restrict__ count_ptr,
                                                      int64_t* __restrict__ counters, int cnt_slot) {
    __shared__ double s_best[8];
    __shared__ int s_idx[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int count = *count_ptr;
    if (blockIdx.x == 0 && threadIdx.x == 0 && counters != nullptr) {
        atomicAdd((unsigned long long*)(counters + cnt_slot), (unsigned long long)count);
        atomicAdd((unsigned long long*)(counters + PARK_CNT_FULL_RESCORE), (unsigned long long)count);
    }
    for (int e = blockIdx.x; e < count; e += gridDim.x) {
        const int gr = rows[e];
        const int bh = gr / N;
        const T* x = X + (size_t)gr * D;
        double xv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = lane + 32 * u;
            xv[u] = j < D ? Elem<T>::to_double(x, j) : 0.0;
        }
        auto partial = [&](int k) -> double {  // this lane's share of distance k
            double s = 0.0;
            if (METRIC) {
                const double* w = w64 + ((size_t)bh * K + k) * D;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = lane + 32 * u;
                    if (j < D) s = __fma_rn(xv[u], w[j], s);
                }
            } else {
                const T* c = C + ((size_t)bh * K + k) * D;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = lane + 32 * u;
                    if (j < D) {
                        const double d = xv[u] - Elem<T>::to_double(c, j);
                        s = __fma_rn(d, d, s);
                    }
                }
            }
            return s;
        };
        double bd = __longlong_as_double(0x7ff0000000000000ll);
        int best = K;
        for (int k = warp; k < K; k += 16) {  // centroids k and k + 8 in flight together
            const int k2 = k + 8;
            double s1 = partial(k), s2 = k2 < K ? partial(k2) : 0.0;
            s1 = warp_sum(s1);
            s2 = warp_sum(s2);
            const double d1 = METRIC ? b64[(size_t)bh * K + k] - 2.0 * s1 : s1;
            if (d1 < bd) {
                bd = d1;
                best = k;
            }
            if (k2 < K) {
                const double d2 = METRIC ? b64[(size_t)bh * K + k2] - 2.0 * s2 : s2;
                if (d2 < bd) {  // k2 > every index seen so far by this warp
                    bd = d2;
                    best = k2;
                }
            }
        }
        if (lane == 0) {
            s_best[warp] = bd;
            s_idx[warp] = best;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            double b = s_best[0];
            int bi = s_idx[0];
            for (int q = 1; q < 8; ++q)
                if (s_best[q] < b || (s_best[q] == b && s_idx[q] < bi)) {
                    b = s_best[q];
                    bi = s_idx[q];
                }
            labels[gr] = bi;
        }
        __syncthreads();
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
    const int fb = num_sms * 4;
    if (dtype == PARK_BF16) {
        if (metric)
            k_rescore_full<bf16_t, true><<<fb, 256, 0, st>>>((const bf16_t*)X, (const bf16_t*)C, w64, b64, N, D, K,
                                                             labels, lists.full_row, lists.counts + 1, counters,
                                                             cnt_slot);
        else
            k_rescore_full<bf16_t, false><<<fb, 256, 0, st>>>((const bf16_t*)X, (const bf16_t*)C, w64, b64, N, D, K,
                                                              labels, lists.full_row, lists.counts + 1, counters,
                                                              cnt_slot);
    } else {
        if (metric)
            k_rescore_full<float, true><<<fb, 256, 0, st>>>((const float*)X, (const float*)C, w64, b64, N, D, K,
                                                            labels, lists.full_row, lists.counts + 1, counters,
                                                            cnt_slot);
        else
            k_rescore_full<float, false><<<fb, 256, 0, st>>>((const float*)X, (const float*)C, w64, b64, N, D, K,
                                                             labels, lists.full_row, lists.counts + 1, counters,
                                                             cnt_slot);
    }
    PARK_TRY_LAUNCH("k_rescore_full", st);
    return PARK_OK;
}

}  // namespace park
