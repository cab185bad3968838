// K-means assign step: a(i) = argmin_k D(x_i, c_k), ties to the lowest k.
//
// Fast path (bf16 inputs): one tensor-core GEMM gives float scores
//   s~_k = bias_k - 2 x . w_k      (Euclidean: w = c, bias = ||c||^2;
//                                  QRKC: w = M c as bf16 hi+lo, bias = c^T M c)
// which equal D(x, c_k) - x^T M x up to a rigorous per-row error bound beta.
// The epilogue keeps the three smallest scores per row.  The winner is
// certified when the runner-up is more than 2 beta above it; otherwise the row
// is listed for a float64 rescore of the two candidates (third score more than
// 2 beta away) or of every centroid.  Float64 rescoring decides all listed
// rows, so labels agree with a float64 evaluation of the definition.
#include "kernels.h"
#include "mma_sync.cuh"

namespace park {

namespace {
__device__ __forceinline__ void top3_insert(float (&v)[3], int (&id)[3], float s, int k) {
    if (s < v[2]) {
        if (s < v[1]) {
            v[2] = v[1];
            id[2] = id[1];
            if (s < v[0]) {
                v[1] = v[0];
                id[1] = id[0];
                v[0] = s;
                id[0] = k;
            } else {
                v[1] = s;
                id[1] = k;
            }
        } else {
            v[2] = s;
            id[2] = k;
        }
    }
}
}  // namespace

// grid (ceil(N/128), BH), 256 threads: 8 warps x 16 rows.  Centroid operands
// stream through shared memory in chunks of 64 (cp.async, double buffered).
template <int KW>
__global__ __launch_bounds__(256, 2) void k_assign_mma(const uint16_t* __restrict__ X,
                                                       const uint16_t* __restrict__ W,
                                                       const float* __restrict__ bias,
                                                       const float* __restrict__ xnorm,
                                                       const float* __restrict__ wmax,
                                                       const float* __restrict__ bmax, float gamma, int N, int K,
                                                       int32_t* __restrict__ labels, Lists lists) {
    constexpr int D = 128;
    constexpr int CH = 64;
    constexpr int LDS = KW + 8;  // padded row: conflict-free ldmatrix
    extern __shared__ __align__(16) uint16_t smem[];
    uint16_t* Ws = smem;                                          // [2][CH][LDS]
    float* Bs = reinterpret_cast<float*>(smem + 2 * CH * LDS);    // [2][CH]

    const int bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const uint16_t* Xh = X + (size_t)bh * N * D;
    const uint16_t* Wh = W + (size_t)bh * K * KW;
    const float* Bh = bias + (size_t)bh * K;

    const int row0 = blockIdx.x * 128 + warp * 16 + g, row1 = row0 + 8;
    uint32_t a[8][4];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        int c0 = kk * 16 + 2 * tq;
        a[kk][0] = row0 < N ? ld_u32(Xh + (size_t)row0 * D + c0) : 0u;
        a[kk][1] = row1 < N ? ld_u32(Xh + (size_t)row1 * D + c0) : 0u;
        a[kk][2] = row0 < N ? ld_u32(Xh + (size_t)row0 * D + c0 + 8) : 0u;
        a[kk][3] = row1 < N ? ld_u32(Xh + (size_t)row1 * D + c0 + 8) : 0u;
    }

    float v[2][3];
    int id[2][3];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int t = 0; t < 3; ++t) {
            v[r][t] = __int_as_float(0x7f800000);
            id[r][t] = 0;
        }

    const int nchunks = (K + CH - 1) / CH;
    auto load_chunk = [&](int c, int stg) {
        int base = c * CH;
        for (int e = threadIdx.x; e < CH * KW / 8; e += 256) {
            int rr = e / (KW / 8), pc = e - rr * (KW / 8);
            int ci = base + rr;
            const uint16_t* src = Wh + (size_t)(ci < K ? ci : K - 1) * KW + pc * 8;
            cp_async16(Ws + (stg * CH + rr) * LDS + pc * 8, src, ci < K ? 16 : 0);
        }
        if (threadIdx.x < CH) {
            int ci = base + threadIdx.x;
            Bs[stg * CH + threadIdx.x] = ci < K ? Bh[ci] : __int_as_float(0x7f800000);
        }
    };

    load_chunk(0, 0);
    cp_async_commit();
    for (int c = 0; c < nchunks; ++c) {
        const int stg = c & 1;
        if (c + 1 < nchunks) load_chunk(c + 1, stg ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();

        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[nt][j] = 0.f;
        const uint16_t* Wst = Ws + stg * CH * LDS;
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int kk = 0; kk < KW / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                int n = np * 16 + (mi >> 1) * 8 + rr;
                int k = kk * 16 + (mi & 1) * 8;
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(b0, b1, b2, b3, Wst + n * LDS + k);
                mma_bf16_16816(acc[2 * np], a[kk & 7], b0, b1);
                mma_bf16_16816(acc[2 * np + 1], a[kk & 7], b2, b3);
            }
        }
        const float* Bst = Bs + stg * CH;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int cl = nt * 8 + 2 * tq + (j & 1);
                int col = c * CH + cl;
                if (col < K) {
                    float s = fmaf(-2.f, acc[nt][j], Bst[cl]);
                    if (j < 2)
                        top3_insert(v[0], id[0], s, col);
                    else
                        top3_insert(v[1], id[1], s, col);
                }
            }
        __syncthreads();
    }

    // merge the four lanes that share a row
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
            float ov[3];
            int oi[3];
#pragma unroll
            for (int t = 0; t < 3; ++t) {
                ov[t] = __shfl_xor_sync(0xffffffffu, v[r][t], off);
                oi[t] = __shfl_xor_sync(0xffffffffu, id[r][t], off);
            }
#pragma unroll
            for (int t = 0; t < 3; ++t) top3_insert(v[r], id[r], ov[t], oi[t]);
        }

    if (tq == 0) {
        const float wm = wmax[bh], bm = bmax[bh];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            int row = r ? row1 : row0;
            if (row >= N) continue;
            size_t gr = (size_t)bh * N + row;
            float beta = gamma * xnorm[gr] * wm + 4.8e-7f * bm + 1e-30f;
            float tb = 2.f * beta;
            labels[gr] = id[r][0];
            if (!(v[r][1] - v[r][0] > tb)) {
                if (v[r][2] - v[r][0] > tb) {
                    int pos = atomicAdd(lists.counts + 0, 1);
                    lists.pair_row[pos] = (int32_t)gr;
                    lists.pair_cand[pos] = id[r][1];
                } else {
                    int pos = atomicAdd(lists.counts + 1, 1);
                    lists.full_row[pos] = (int32_t)gr;
                }
            }
        }
    }
}

int launch_assign_mma(const void* X, int BH, int N, int K, const CentroidOps& ops, const float* xnorm,
                      float gamma, int32_t* labels, Lists lists, cudaStream_t st) {
    dim3 grid((N + 127) / 128, BH);
    if (ops.kw != 128 && ops.kw != 256) return PARK_ERR_UNSUPPORTED;
    if (ops.kw == 256)
        cudaFuncSetAttribute(k_assign_mma<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             2 * 64 * (256 + 8) * 2 + 2 * 64 * 4);
    ::park::prof_begin(st);
    if (ops.kw == 128) {
        size_t sm = 2 * 64 * (128 + 8) * 2 + 2 * 64 * 4;
        k_assign_mma<128><<<grid, 256, sm, st>>>((const uint16_t*)X, ops.w, ops.bias32, xnorm, ops.wmax, ops.bmax,
                                                 gamma, N, K, labels, lists);
    } else if (ops.kw == 256) {
        size_t sm = 2 * 64 * (256 + 8) * 2 + 2 * 64 * 4;
        k_assign_mma<256><<<grid, 256, sm, st>>>((const uint16_t*)X, ops.w, ops.bias32, xnorm, ops.wmax, ops.bmax,
                                                 gamma, N, K, labels, lists);
    }
    PARK_TRY_LAUNCH("k_assign_mma", st);
    return PARK_OK;
}

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
