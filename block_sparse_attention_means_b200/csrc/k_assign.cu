// K-means assign step: a(i) = argmin_k D(x_i, c_k), ties to the lowest k.
//
// Fast path (bf16 inputs, k_assign_tc.cu): one tensor-core GEMM gives float scores
//   s~_k = bias_k - 2 x . w_k      (Euclidean: w = c, bias = ||c||^2;
//                                  QRKC: w = M c as bf16 hi+lo, bias = c^T M c)
// which equal D(x, c_k) - x^T M x up to a rigorous per-row error bound beta.
// The epilogue keeps the three smallest scores per row.  The winner is
// certified when the runner-up is more than 2 beta above it; otherwise the row
// is listed for a float64 rescore of the two candidates (third score more than
// 2 beta away) or of every centroid.  Float64 rescoring decides all listed
// rows, so labels agree with a float64 evaluation of the definition.
#include "kernels.h"

namespace park {


// ---------------------------------------------------------------- float64 rescore
// One warp per listed row.  mode 0: the row's two candidates (current label and
// runner-up); mode 1: every centroid; mode 2: every row of every head against
// every centroid (the float32 input path, which has no tensor-core filter).
// Euclidean distance: sum_j (x_j - c_j)^2.  QRKC: c^T M c - 2 x . (M c), the
// distance minus the row constant x^T M x.  Ties go to the lowest index.
template <typename T, bool METRIC>
__global__ void k_recheck(const T* __restrict__ X, const T* __restrict__ C, const double* __restrict__ w64,
                          const double* __restrict__ b64, int N, int D, int K, int32_t* __restrict__ labels,
                          const int32_t* __restrict__ rows, const int32_t* __restrict__ cand,
                          const int32_t* __restrict__ count_ptr, int mode, int total_rows,
                          int64_t* __restrict__ counters, int cnt_slot) {
    const int lane = threadIdx.x & 31;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    const int count = mode == 2 ? total_rows : *count_ptr;
    if (blockIdx.x == 0 && threadIdx.x == 0 && counters != nullptr && mode != 2) {
        atomicAdd((unsigned long long*)(counters + cnt_slot), (unsigned long long)count);
        if (mode == 1) atomicAdd((unsigned long long*)(counters + PARK_CNT_FULL_RESCORE), (unsigned long long)count);
    }
    for (int e = gw; e < count; e += nw) {
        const int gr = mode == 2 ? e : rows[e];
        const int bh = gr / N;
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
        int best;
        if (mode == 0) {
            int k1 = labels[gr], k2 = cand[e];
            double d1 = dist(k1), d2 = dist(k2);
            best = (d2 < d1 || (d2 == d1 && k2 < k1)) ? k2 : k1;
        } else {
            double bd = __longlong_as_double(0x7ff0000000000000ll);
            best = 0;
            for (int k = 0; k < K; ++k) {
                double d = dist(k);
                if (d < bd) {
                    bd = d;
                    best = k;
                }
            }
        }
        if (lane == 0) labels[gr] = best;
    }
}

int launch_recheck(const void* X, int dtype, int BH, int N, int D, int K, const void* C, const double* w64,
                   const double* b64, int32_t* labels, Lists lists, int all_rows, int num_sms,
                   int64_t* counters, int cnt_slot, cudaStream_t st) {
    if (D > 128) return PARK_ERR_UNSUPPORTED;
    const bool metric = w64 != nullptr;
    const int blocks = num_sms * 8, threads = 256;
    const int total = BH * N;
    auto go = [&](int mode, const int32_t* rows, const int32_t* cand, const int32_t* cnt) {
        ::park::prof_begin(st);
        if (dtype == PARK_BF16) {
            if (metric)
                k_recheck<bf16_t, true><<<blocks, threads, 0, st>>>((const bf16_t*)X, (const bf16_t*)C, w64, b64, N,
                                                                   D, K, labels, rows, cand, cnt, mode, total,
                                                                   counters, cnt_slot);
            else
                k_recheck<bf16_t, false><<<blocks, threads, 0, st>>>((const bf16_t*)X, (const bf16_t*)C, w64, b64,
                                                                    N, D, K, labels, rows, cand, cnt, mode, total,
                                                                    counters, cnt_slot);
        } else {
            if (metric)
                k_recheck<float, true><<<blocks, threads, 0, st>>>((const float*)X, (const float*)C, w64, b64, N, D,
                                                                  K, labels, rows, cand, cnt, mode, total,
                                                                  counters, cnt_slot);
            else
                k_recheck<float, false><<<blocks, threads, 0, st>>>((const float*)X, (const float*)C, w64, b64, N,
                                                                   D, K, labels, rows, cand, cnt, mode, total,
                                                                   counters, cnt_slot);
        }
    };
    if (all_rows) {
        go(2, nullptr, nullptr, nullptr);
        PARK_TRY_LAUNCH("k_recheck", st);
    } else {
        go(0, lists.pair_row, lists.pair_cand, lists.counts + 0);
        PARK_TRY_LAUNCH("k_recheck", st);
        go(1, lists.full_row, nullptr, lists.counts + 1);
        PARK_TRY_LAUNCH("k_recheck", st);
    }
    return PARK_OK;
}

}  // namespace park
