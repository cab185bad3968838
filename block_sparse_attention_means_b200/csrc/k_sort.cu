// Stable counting sort of tokens by cluster label (perm, offsets) and the
// exact K-means centroid update.
//
// Sort: tokens are split into chunks of 1024.  (1) per-chunk label histogram
// in shared memory; (2) the [label][chunk] table becomes start positions
// (label-major, so clusters are contiguous and chunks keep token order); (3)
// each chunk ranks its tokens among equal labels in token order (warp match +
// warps in sequence) and scatters them.  The result equals a stable argsort of
// the labels.
//
// Update: one CTA per (cluster, head) sums its members' rows exactly in 128-bit
// fixed point (x * 2^64; integer sums are exact and independent of order),
// converts the exact sum to float64 with one correct rounding, divides by the
// member count in IEEE float64 and rounds to the storage dtype (nearest, ties
// to even).  Empty clusters keep their centroid.
#include "kernels.h"

namespace park {

constexpr int SORT_CHUNK = 1024;

__global__ void k_label_hist(const int32_t* __restrict__ labels, int N, int K, int nchunks,
                             int32_t* __restrict__ hist) {
    extern __shared__ int32_t cnt[];
    int c = blockIdx.x, bh = blockIdx.y;
    for (int k = threadIdx.x; k < K; k += blockDim.x) cnt[k] = 0;
    __syncthreads();
    int i0 = c * SORT_CHUNK, i1 = min(N, i0 + SORT_CHUNK);
    const int32_t* lab = labels + (size_t)bh * N;
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) atomicAdd(&cnt[lab[i]], 1);
    __syncthreads();
    int32_t* h = hist + (size_t)bh * K * nchunks;
    for (int k = threadIdx.x; k < K; k += blockDim.x) h[(size_t)k * nchunks + c] = cnt[k];
}

// Positions, in two steps that keep every SM busy.  (2a) one warp per (label,
// head) turns its row hist[k][*] into exclusive positions within the label and
// writes the label's size to offsets[k]; (2b) one CTA per head turns the sizes
// into exclusive starts, offsets[K] = N.  A token's position is offsets[label]
// + hist[label][chunk] + its rank in the chunk.
__global__ __launch_bounds__(256) void k_label_rowscan(int32_t* __restrict__ hist, int K, int nchunks,
                                                       int32_t* __restrict__ offsets) {
    const int lane = threadIdx.x & 31;
    const int k = blockIdx.x * 8 + (threadIdx.x >> 5), bh = blockIdx.y;
    if (k >= K) return;
    int32_t* h = hist + ((size_t)bh * K + k) * nchunks;
    const int seg = (nchunks + 31) / 32, b0 = lane * seg, b1 = min(nchunks, b0 + seg);
    int loc = 0;
    for (int e = b0; e < b1; ++e) loc += h[e];
    int incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    int run = incl - loc;
    for (int e = b0; e < b1; ++e) {
        const int v = h[e];
        h[e] = run;
        run += v;
    }
    if (lane == 31) offsets[(size_t)bh * (K + 1) + k] = incl;
}

__global__ __launch_bounds__(1024) void k_label_scan(int N, int K, int32_t* __restrict__ offsets) {
    __shared__ int32_t wsum[32];
    const int bh = blockIdx.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
    int32_t* off = offsets + (size_t)bh * (K + 1);
    const int seg = (K + 1023) / 1024, b0 = t * seg, b1 = min(K, b0 + seg);
    int loc = 0;
    for (int e = b0; e < b1; ++e) loc += off[e];
    int incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    if (w == 0) {
        const int x = wsum[lane];
        int xi = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, xi, o);
            if (lane >= o) xi += y;
        }
        wsum[lane] = xi - x;
    }
    __syncthreads();
    int run = wsum[w] + incl - loc;
    for (int e = b0; e < b1; ++e) {
        const int v = off[e];
        off[e] = run;
        run += v;
    }
    if (t == 0) off[K] = N;
}

__global__ __launch_bounds__(1024) void k_label_scatter(const int32_t* __restrict__ labels, int N, int K,
                                                        int nchunks, const int32_t* __restrict__ hist,
                                                        const int32_t* __restrict__ offsets,
                                                        int32_t* __restrict__ perm) {
    extern __shared__ int32_t run[];  // [K] tokens already placed per label in this chunk
    int c = blockIdx.x, bh = blockIdx.y;
    for (int k = threadIdx.x; k < K; k += blockDim.x) run[k] = 0;
    __syncthreads();
    int i = c * SORT_CHUNK + threadIdx.x;
    bool valid = i < N;
    int lab = valid ? labels[(size_t)bh * N + i] : -1;
    int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned peers = __match_any_sync(0xffffffffu, lab);
    unsigned lower = peers & ((1u << lane) - 1u);
    int rank = __popc(lower);
    bool leader = lower == 0u;
    int pos = 0;
    for (int w = 0; w < 32; ++w) {
        if (warp == w) {
            int base = valid ? run[lab] : 0;
            __syncwarp();
            if (valid && leader) run[lab] = base + __popc(peers);
            if (valid) pos = offsets[(size_t)bh * (K + 1) + lab] + hist[((size_t)bh * K + lab) * nchunks + c] + base + rank;
        }
        __syncthreads();
    }
    if (valid) perm[(size_t)bh * N + pos] = i;
}

int launch_label_sort(const int32_t* labels, int BH, int N, int K, int32_t* hist, int nchunks, int32_t* perm,
                      int32_t* offsets, cudaStream_t st) {
    size_t sm = (size_t)K * sizeof(int32_t);
    if (sm > 48 * 1024) {
        cudaFuncSetAttribute(k_label_hist, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        cudaFuncSetAttribute(k_label_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    }
    dim3 g(nchunks, BH);
    ::park::prof_begin(st);
    k_label_hist<<<g, 256, sm, st>>>(labels, N, K, nchunks, hist);
    PARK_TRY_LAUNCH("k_label_hist", st);
    ::park::prof_begin(st);
    k_label_rowscan<<<dim3((K + 7) / 8, BH), 256, 0, st>>>(hist, K, nchunks, offsets);
    PARK_TRY_LAUNCH("k_label_rowscan", st);
    ::park::prof_begin(st);
    k_label_scan<<<BH, 1024, 0, st>>>(N, K, offsets);
    PARK_TRY_LAUNCH("k_label_scan", st);
    ::park::prof_begin(st);
    k_label_scatter<<<g, 1024, sm, st>>>(labels, N, K, nchunks, hist, offsets, perm);
    PARK_TRY_LAUNCH("k_label_scatter", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- update
// 128 threads.  Each thread owns one 16-byte piece of a row: VEC elements at
// piece p = t % CPR, and rows s, s + RPI, ... of the cluster (s = t / CPR).
// The sum is exact: every element is taken as the integer x * 2^64 (exact for
// the whole range precondition) and summed in a signed 128-bit integer.
// bf16 elements with 2^-20 <= |x| < 2^16 -- all of them on unit-scale data --
// go through a float64 partial sum per element that is exact for 1024 rows
// (such values are multiples of 2^-27 below 2^16, so 1024 of them need at most
// 53 bits); every 1024 rows it moves, as the integer part * 2^27 (below 2^53),
// into an int64 sum (at most 128 moves per thread: below 2^60), which counts
// x * 2^64 in units of 2^37.  A piece holding any other element (rare) adds
// all its elements as x * 2^64 directly to 128-bit sums kept in shared memory.  float32 elements all take the 128-bit
// path, in registers.
// Adds the eight bf16 elements of a 16-byte piece, as x * 2^64, to 128-bit sums.
__device__ __noinline__ void update_slow_piece(uint4 v, unsigned long long* lo, long long* hi) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        unsigned long long l = lo[e];
        long long h = hi[e];
        fixed64_add(l, h, (e & 1) ? (w[e >> 1] & 0xffff0000u) : (w[e >> 1] << 16));
        lo[e] = l;
        hi[e] = h;
    }
}

template <typename T>
__global__ __launch_bounds__(128) void k_update(const T* __restrict__ X, const int32_t* __restrict__ perm,
                                                const int32_t* __restrict__ offsets, int N, int D, int K,
                                                T* __restrict__ C) {
    constexpr int VEC = 16 / sizeof(T);
    constexpr bool BF16 = sizeof(T) == 2;
    extern __shared__ long long red[];  // [2][RPI][D]: high and low words of the 128-bit sums
    __shared__ unsigned long long slow_lo[BF16 ? 128 * VEC : 1];
    __shared__ long long slow_hi[BF16 ? 128 * VEC : 1];
    int k = blockIdx.x, bh = blockIdx.y;
    const int32_t* off = offsets + (size_t)bh * (K + 1);
    int start = off[k], n = off[k + 1] - start;
    if (n == 0) return;  // empty cluster keeps its centroid
    const int CPR = D / VEC, RPI = 128 / CPR;
    int t = threadIdx.x, piece = t % CPR, slot = t / CPR;
    long long acc_hi[BF16 ? 1 : VEC];             // float32: 128-bit sums in registers
    unsigned long long acc_lo[BF16 ? 1 : VEC];
    long long mid[BF16 ? VEC : 1];                // bf16: flushed partials, units of 2^37
    double part[BF16 ? VEC : 1];
#pragma unroll
    for (int e = 0; e < (BF16 ? 1 : VEC); ++e) {
        acc_hi[e] = 0;
        acc_lo[e] = 0;
    }
#pragma unroll
    for (int e = 0; e < (BF16 ? VEC : 1); ++e) {
        mid[e] = 0;
        part[e] = 0.0;
    }
    if (BF16) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            slow_lo[t * VEC + e] = 0ull;
            slow_hi[t * VEC + e] = 0;
        }
    }
    const int32_t* pm = perm + (size_t)bh * N + start;
    const T* Xh = X + (size_t)bh * N * D;
    int rows_in_part = 0;
    auto flush = [&]() {
        if (BF16) {
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                mid[e] += __double2ll_rn(ldexp(part[e], 27));  // exact: a multiple of 2^-27 below 2^26
                part[e] = 0.0;
            }
        }
        rows_in_part = 0;
    };
    auto add_piece = [&](const uint4& v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        if (BF16) {
            // the common case, decided once per 16-byte piece with 16-bit SIMD compares:
            // every element is 0 or has 2^-20 <= |x| < 2^16 (biased exponent 107..142)
            uint32_t bad = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t ex = (w[q] >> 7) & 0x00FF00FFu;
                const uint32_t in = __vcmpgeu2(ex, 0x006B006Bu) & __vcmpleu2(ex, 0x008E008Eu);
                bad |= ~(in | __vcmpeq2(w[q] & 0x7FFF7FFFu, 0u));
            }
            if (bad == 0) {
#pragma unroll
                for (int e = 0; e < VEC; ++e)
                    part[e] += (double)__uint_as_float((e & 1) ? (w[e >> 1] & 0xffff0000u) : (w[e >> 1] << 16));
            } else {  // rare: the whole piece goes to the 128-bit sums, out of line
                update_slow_piece(v, slow_lo + t * VEC, slow_hi + t * VEC);
            }
            if (++rows_in_part == 1024) flush();
        } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) fixed64_add(acc_lo[e], acc_hi[e], w[e]);
        }
    };
    if (slot < RPI) {
        // four member rows in flight per thread (integer sums: the order does not matter)
        int j = slot;
        for (; j + 3 * RPI < n; j += 4 * RPI) {
            int tok[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) tok[u] = pm[j + u * RPI];
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = *reinterpret_cast<const uint4*>(Xh + (size_t)tok[u] * D + piece * VEC);
#pragma unroll
            for (int u = 0; u < 4; ++u) add_piece(v[u]);
        }
        for (; j < n; j += RPI) add_piece(*reinterpret_cast<const uint4*>(Xh + (size_t)pm[j] * D + piece * VEC));
        flush();
    }
    long long* red_hi = red;
    long long* red_lo = red + RPI * D;
    if (slot < RPI) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            unsigned long long lo;
            long long hi;
            if (BF16) {  // mid * 2^37 plus the directly added elements
                lo = (unsigned long long)mid[e] << 37;
                hi = mid[e] >> 27;
                acc128_add(lo, hi, slow_lo[t * VEC + e], slow_hi[t * VEC + e]);
            } else {
                lo = acc_lo[e];
                hi = acc_hi[e];
            }
            red_hi[slot * D + piece * VEC + e] = hi;
            red_lo[slot * D + piece * VEC + e] = (long long)lo;
        }
    }
    __syncthreads();
    if (t < D) {
        long long sh = 0;
        unsigned long long sl = 0;
        for (int q = 0; q < RPI; ++q) acc128_add(sl, sh, (unsigned long long)red_lo[q * D + t], red_hi[q * D + t]);
        // one correct rounding of the exact sum to float64, then the IEEE division by n
        const double mean = ldexp(i128_to_double_rn(sh, sl), -64) / (double)n;
        T* c = C + ((size_t)bh * K + k) * D + t;
        if (sizeof(T) == 2)
            reinterpret_cast<uint16_t*>(c)[0] = double_to_bf16_bits(mean);
        else
            reinterpret_cast<float*>(c)[0] = __double2float_rn(mean);
    }
}

int launch_update(const void* X, int dtype, int BH, int N, int D, int K, const int32_t* perm,
                  const int32_t* offsets, void* C, cudaStream_t st) {
    dim3 g(K, BH);
    const int vec = dtype == PARK_BF16 ? 8 : 4;
    if (D % vec || D / vec > 128) return PARK_ERR_UNSUPPORTED;
    ::park::prof_begin(st);
    if (dtype == PARK_BF16) {
        int rpi = 128 / (D / 8);
        k_update<bf16_t><<<g, 128, (size_t)rpi * D * 16, st>>>((const bf16_t*)X, perm, offsets, N, D, K, (bf16_t*)C);
    } else {
        int rpi = 128 / (D / 4);
        k_update<float><<<g, 128, (size_t)rpi * D * 16, st>>>((const float*)X, perm, offsets, N, D, K, (float*)C);
    }
    PARK_TRY_LAUNCH("k_update", st);
    return PARK_OK;
}

}  // namespace park
