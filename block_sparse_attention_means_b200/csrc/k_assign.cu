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
// head.  CTA (s, bh) takes groups of up to eight listed rows of head bh (groups
// s, s + gridDim.x, ...); warp w scores centroids w, w + 8, ... against every row
// of the group (lane l holds elements l, l + 32, l + 64, l + 96 of each row), so
// every centroid operand is read once per group instead of once per row.  Each
// distance is the same float64 expression, summed in the same order, as a
// one-row evaluation; ties go to the lowest index.
constexpr int kRescoreRows = 8;

template <typename T, bool METRIC>
__global__ __launch_bounds__(256) void k_rescore_full(const T* __restrict__ X, const T* __restrict__ C,
                                                      const double* __restrict__ w64, const double* __restrict__ b64,
                                                      int N, int D, int K, int32_t* __restrict__ labels,
                                                      const int32_t* __restrict__ rows,
                                                      const int32_t* __restrict__ counts,
                                                      int64_t* __restrict__ counters, int cnt_slot) {
    constexpr int R = kRescoreRows;
    __shared__ double s_best[8][R];
    __shared__ int s_idx[8][R];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int bh = blockIdx.y;
    const int count = counts[bh];
    if (blockIdx.x == 0 && threadIdx.x == 0 && counters != nullptr && count > 0) {
        atomicAdd((unsigned long long*)(counters + cnt_slot), (unsigned long long)count);
        atomicAdd((unsigned long long*)(counters + PARK_CNT_FULL_RESCORE), (unsigned long long)count);
    }
    const int32_t* list = rows + (size_t)bh * N;
    for (int g0 = blockIdx.x * R; g0 < count; g0 += gridDim.x * R) {
        const int nr = min(R, count - g0);
        double xv[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int gr = list[g0 + (r < nr ? r : 0)];  // rows past the group repeat its first row
            const T* x = X + (size_t)gr * D;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = lane + 32 * u;
                xv[r][u] = j < D ? Elem<T>::to_double(x, j) : 0.0;
            }
        }
        double bd[R];
        int best[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            bd[r] = __longlong_as_double(0x7ff0000000000000ll);
            best[r] = K;
        }
        // four centroids per warp step (k, k + 8, k + 16, k + 24): their operand loads
        // are in flight together
        constexpr int U = 4;
        for (int k0 = warp; k0 < K; k0 += 8 * U) {
            double cv[U][4], bk[U];
#pragma unroll
            for (int v = 0; v < U; ++v) {
                const int k = k0 + 8 * v;
                const bool kin = k < K;
                if (METRIC) {
                    const double* w = w64 + ((size_t)bh * K + (kin ? k : 0)) * D;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = lane + 32 * u;
                        cv[v][u] = (kin && j < D) ? w[j] : 0.0;
                    }
                    bk[v] = kin ? b64[(size_t)bh * K + k] : 0.0;
                } else {
                    const T* c = C + ((size_t)bh * K + (kin ? k : 0)) * D;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = lane + 32 * u;
                        cv[v][u] = (kin && j < D) ? Elem<T>::to_double(c, j) : 0.0;
                    }
                    bk[v] = 0.0;
                }
            }
#pragma unroll
            for (int v = 0; v < U; ++v) {
                const int k = k0 + 8 * v;
                if (k >= K) break;  // uniform over the warp
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    double s = 0.0;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = lane + 32 * u;
                        if (j < D) {
                            if (METRIC) {
                                s = __fma_rn(xv[r][u], cv[v][u], s);
                            } else {
                                const double d = xv[r][u] - cv[v][u];
                                s = __fma_rn(d, d, s);
                            }
                        }
                    }
                    s = warp_sum(s);
                    const double d = METRIC ? bk[v] - 2.0 * s : s;
                    if (d < bd[r]) {  // k grows within the warp: the first of equal distances stays
                        bd[r] = d;
                        best[r] = k;
                    }
                }
            }
        }
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                s_best[warp][r] = bd[r];
                s_idx[warp][r] = best[r];
            }
        }
        __syncthreads();
        if (threadIdx.x < nr) {
            const int r = threadIdx.x;
            double b = s_best[0][r];
            int bi = s_idx[0][r];
            for (int q = 1; q < 8; ++q)
                if (s_best[q][r] < b || (s_best[q][r] == b && s_idx[q][r] < bi)) {
                    b = s_best[q][r];
                    bi = s_idx[q][r];
                }
            labels[list[g0 + r]] = bi;
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
    // per head: enough CTAs for about four per SM over all heads
    const dim3 fb((unsigned)std::max(1, (num_sms * 4 + BH - 1) / BH), (unsigned)BH);
    if (dtype == PARK_BF16) {
        if (metric)
            k_rescore_full<bf16_t, true><<<fb, 256, 0, st>>>((const bf16_t*)X, (const bf16_t*)C, w64, b64, N, D, K,
                                                             labels, lists.full_row, lists.counts, counters,
                                                             cnt_slot);
        else
            k_rescore_full<bf16_t, false><<<fb, 256, 0, st>>>((const bf16_t*)X, (const bf16_t*)C, w64, b64, N, D, K,
                                                              labels, lists.full_row, lists.counts, counters,
                                                              cnt_slot);
    } else {
        if (metric)
            k_rescore_full<float, true><<<fb, 256, 0, st>>>((const float*)X, (const float*)C, w64, b64, N, D, K,
                                                            labels, lists.full_row, lists.counts, counters,
                                                            cnt_slot);
        else
            k_rescore_full<float, false><<<fb, 256, 0, st>>>((const float*)X, (const float*)C, w64, b64, N, D, K,
                                                             labels, lists.full_row, lists.counts, counters,
                                                             cnt_slot);
    }
    PARK_TRY_LAUNCH("k_rescore_full", st);
    return PARK_OK;
}

}  // namespace park
