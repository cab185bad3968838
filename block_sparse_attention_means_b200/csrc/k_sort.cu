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

// (3), for K <= kScatterMaxK: each warp's leaders record the counts of their
// labels in a [warp][label] table in shared memory; one pass per label turns the
// table into the number of earlier tokens of the chunk with that label (the
// warps in order), so the ranks need three block barriers instead of one per
// warp.
constexpr int kScatterMaxK = 1536;

__global__ __launch_bounds__(1024) void k_label_scatter_tab(const int32_t* __restrict__ labels, int N, int K,
                                                            int KP, int nchunks, const int32_t* __restrict__ hist,
                                                            const int32_t* __restrict__ offsets,
                                                            int32_t* __restrict__ perm) {
    extern __shared__ uint16_t tab[];  // [32][KP]: counts, then exclusive starts over the warps
    const int c = blockIdx.x, bh = blockIdx.y;
    uint32_t* tab32 = reinterpret_cast<uint32_t*>(tab);
    for (int e = threadIdx.x; e < 16 * KP; e += blockDim.x) tab32[e] = 0u;  // 32 KP uint16 (KP even)
    const int i = c * SORT_CHUNK + threadIdx.x;
    const bool valid = i < N;
    const int lab = valid ? labels[(size_t)bh * N + i] : -1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned peers = __match_any_sync(0xffffffffu, lab);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    __syncthreads();
    if (valid && rank == 0) tab[warp * KP + lab] = (uint16_t)__popc(peers);
    __syncthreads();
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        uint32_t run = 0;
#pragma unroll
        for (int h = 0; h < 32; h += 16) {  // sixteen loads in flight
            uint32_t v[16];
#pragma unroll
            for (int w = 0; w < 16; ++w) v[w] = tab[(h + w) * KP + k];
#pragma unroll
            for (int w = 0; w < 16; ++w) {
                tab[(h + w) * KP + k] = (uint16_t)run;
                run += v[w];
            }
        }
    }
    __syncthreads();
    if (valid) {
        const int pos = offsets[(size_t)bh * (K + 1) + lab] + hist[((size_t)bh * K + lab) * nchunks + c] +
                        tab[warp * KP + lab] + rank;
        perm[(size_t)bh * N + pos] = i;
    }
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
    if (K <= kScatterMaxK) {
        const int KP = (K + 1) & ~1;  // even row pitch: the table is zeroed in 32-bit words
        const size_t tsm = (size_t)32 * KP * sizeof(uint16_t);
        if (tsm > 48 * 1024)
            cudaFuncSetAttribute(k_label_scatter_tab, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
        k_label_scatter_tab<<<g, 1024, tsm, st>>>(labels, N, K, KP, nchunks, hist, offsets, perm);
    } else {
        k_label_scatter<<<g, 1024, sm, st>>>(labels, N, K, nchunks, hist, offsets, perm);
    }
    PARK_TRY_LAUNCH("k_label_scatter", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- update
// 128 threads.  Each thread owns one 16-byte piece of a row: VEC elements at
// piece p = t % CPR, and rows s, s + RPI, ... of the cluster (s = t / CPR).
// Every sum is exact: the integer x * 2^64, summed in a signed 128-bit integer
// (exact over the whole range precondition; fixed64_add).  On a bf16 head
// without elements of magnitude 2^16 or more (the input check flags the others;
// unit-scale data has none) the same integer is reached faster:
//   * rows without a nonzero element below 2^-20 (the input check flags the
//     others, one byte per row) go into float64 partial sums per element,
//     exact for 1024 rows (every element is a multiple of 2^-27 below 2^16:
//     1024 of them need at most 53 bits), moved every 1024 rows into an int64
//     sum of x * 2^27 (at most 128 moves per thread: below 2^60);
//   * a flagged row's piece goes, out of line, to int64 sums in shared memory:
//     x * 2^47 for its elements below 2^-20 (below 2^27 inside the range),
//     x * 2^27 for the others.
// Other heads, and float32 inputs, take the general path, out of line.

// The general path of one thread: 128-bit sums of its VEC elements over rows
// slot, slot + RPI, ..., written to red_hi / red_lo.
template <typename T>
__device__ __noinline__ void update_exact_rows(const T* __restrict__ Xh, const int32_t* __restrict__ pm, int n,
                                               int D, int piece, int slot, int RPI, long long* red_hi,
                                               long long* red_lo) {
    constexpr int VEC = 16 / sizeof(T);
    long long hi[VEC];
    unsigned long long lo[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        hi[e] = 0;
        lo[e] = 0;
    }
    for (int j = slot; j < n; j += RPI) {
        const uint4 v = *reinterpret_cast<const uint4*>(Xh + (size_t)pm[j] * D + piece * VEC);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            const uint32_t u = sizeof(T) == 2 ? ((e & 1) ? (w[e >> 1] & 0xffff0000u) : (w[e >> 1] << 16)) : w[e];
            fixed64_add(lo[e], hi[e], u);
        }
    }
    const int CPR = D / VEC;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {  // layout [slot][e][piece]
        red_hi[slot * D + e * CPR + piece] = hi[e];
        red_lo[slot * D + e * CPR + piece] = (long long)lo[e];
    }
}

// x * 2^47 of a bf16 element (IEEE-single bits u) with 2^-40 <= |x| < 2^-20:
// the significand m (8 bits with the leading one) shifted by e - 87 (0 .. 19);
// lower exponents (outside the range precondition, reported by the input check)
// are clamped.
__device__ inline long long tiny_fixed47(uint32_t u) {
    const int e = (u >> 23) & 0xFF;
    const long long m = (long long)(0x80u | ((u >> 16) & 0x7Fu));
    const int sh = e - 87;
    const long long v = sh >= 0 ? (m << sh) : (m >> min(-sh, 63));
    return (u & 0x80000000u) ? -v : v;
}

// A piece of a flagged bf16 row: elements below 2^-20 add x * 2^47 to
// tiny[e * stride], the others (2^-20 <= |x| < 2^16 on a head without larger
// values, or 0) add the integer x * 2^27 to norm[e * stride].
__device__ __noinline__ void update_tiny_piece(uint4 v, long long* tiny, long long* norm, int stride) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const uint32_t b = (e & 1) ? (w[e >> 1] & 0xffff0000u) : (w[e >> 1] << 16);
        const uint32_t mag = b & 0x7FFFFFFFu;
        if (mag == 0u) continue;
        if (mag < 0x35800000u) {
            tiny[e * stride] += tiny_fixed47(b);
        } else {  // m << (e - 107): an integer below 2^43
            const int ex = (b >> 23) & 0xFF;
            const long long m = (long long)(0x80u | ((b >> 16) & 0x7Fu)) << min(max(ex - 107, 0), 35);
            norm[e * stride] += (b & 0x80000000u) ? -m : m;
        }
    }
}

constexpr int kUpdStage = 1024;  // member tokens staged in shared memory at a time

// The float64 value of a bf16 element given as IEEE-single bits f (low 16 bits
// zero), for 0 and normal values, built with integer operations: the sign, the
// exponent rebiased by 1023 - 127 and the 7 stored significand bits in the high
// word, a zero low word.  (The float32 -> float64 conversion instruction runs at a
// fraction of the integer rate and bounded the update.)
__device__ __forceinline__ double bf16_bits_to_f64(uint32_t f) {
    const uint32_t mag = f & 0x7FFFFFFFu;
    const uint32_t hi = mag ? (((mag >> 3) + 0x38000000u) | (f & 0x80000000u)) : f;
    return __hiloint2double((int)hi, 0);
}

template <typename T>
__global__ __launch_bounds__(128, 5) void k_update(const T* __restrict__ X, const int32_t* __restrict__ perm,
                                                const int32_t* __restrict__ offsets, int N, int D, int K,
                                                T* __restrict__ C, const int32_t* __restrict__ wide,
                                                const uint8_t* __restrict__ tiny_rows) {
    constexpr int VEC = 16 / sizeof(T);
    extern __shared__ long long red[];  // [2][RPI][D]: high and low words of the 128-bit sums
    __shared__ int32_t stok[sizeof(T) == 2 ? kUpdStage : 1];  // member tokens of the current stage
    int k = blockIdx.x, bh = blockIdx.y;
    const int32_t* off = offsets + (size_t)bh * (K + 1);
    int start = off[k], n = off[k + 1] - start;
    if (n == 0) return;  // empty cluster keeps its centroid
    const int CPR = D / VEC, RPI = 128 / CPR;
    int t = threadIdx.x, piece = t % CPR, slot = t / CPR;
    long long* red_hi = red;
    long long* red_lo = red + RPI * D;
    const int32_t* pm = perm + (size_t)bh * N + start;
    const T* Xh = X + (size_t)bh * N * D;
    // uniform over the CTA
    const bool fast = sizeof(T) == 2 && wide != nullptr && tiny_rows != nullptr && wide[bh] == 0 && RPI * CPR == 128;
    if (!fast) {
        if (slot < RPI) update_exact_rows<T>(Xh, pm, n, D, piece, slot, RPI, red_hi, red_lo);
    } else {
        const uint8_t* trow = tiny_rows + (size_t)bh * N;
        // until the end, red holds the flagged rows' int64 sums element-major ([e][t]:
        // consecutive threads, consecutive words): x * 2^27 in red_hi for their elements of
        // 2^-20 and above, x * 2^47 in red_lo for those below
        long long* norm = red_hi + t;
        long long* tiny = red_lo + t;
        long long acc[VEC];  // x * 2^27: the flushed float64 partial sums
        double part[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            acc[e] = 0;
            part[e] = 0.0;
            norm[e * 128] = 0;
            tiny[e * 128] = 0;
        }
        auto flush = [&]() {
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                acc[e] += __double2ll_rn(part[e] * 0x1p27);  // exact: a multiple of 2^-27 below 2^26
                part[e] = 0.0;
            }
        };
        auto add_fast = [&](const uint4& v) {
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < VEC; ++e)
                part[e] += bf16_bits_to_f64((e & 1) ? (w[e >> 1] & 0xffff0000u) : (w[e >> 1] << 16));
        };
        // The cluster's member tokens are staged in shared memory (kUpdStage at a time,
        // one coalesced load), each with its row's flag in the sign bit (one flag load per
        // row instead of one per 16-byte piece: those cost 40 % of the kernel), so each
        // member row costs one dependent global load; eight rows in flight per thread
        // (integer sums: the order does not matter).  A thread
        // takes kUpdStage / RPI <= 1024 rows per stage: one flush per stage keeps every
        // float64 partial sum within 1024 rows.
        for (int base = 0; base < n; base += kUpdStage) {
            const int cnt = min(kUpdStage, n - base);
            __syncthreads();  // the previous stage's tokens have been read
            for (int i = t; i < cnt; i += blockDim.x) {
                const int tk = pm[base + i];
                stok[i] = trow[tk] ? (tk | (int)0x80000000u) : tk;
            }
            __syncthreads();
            // every batch, the last one included, keeps its eight loads in flight: rows past
            // the stage read as zero, which adds nothing to the exact sums
            for (int j = slot; j < cnt; j += 8 * RPI) {
                uint4 v[8];
                uint32_t fl = 0;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int r = j + u * RPI;
                    v[u] = make_uint4(0u, 0u, 0u, 0u);
                    if (r < cnt) {
                        const int sv = stok[r];
                        const int tk = sv & 0x7FFFFFFF;
                        v[u] = *reinterpret_cast<const uint4*>(Xh + (size_t)tk * D + piece * VEC);
                        fl |= (uint32_t)(sv < 0) << u;
                    }
                }
                if (fl == 0u) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) add_fast(v[u]);
                } else {  // rare
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        if (fl >> u & 1u)
                            update_tiny_piece(v[u], tiny, norm, 128);
                        else
                            add_fast(v[u]);
                    }
                }
            }
            flush();
        }
        long long hv[VEC];
        unsigned long long lv[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            // x * 2^64 = (acc + norm) * 2^37 + tiny * 2^17 as a 128-bit integer (|acc + norm| < 2^61,
            // |tiny| < 2^47)
            const long long a = acc[e] + norm[e * 128];
            lv[e] = (unsigned long long)a << 37;
            hv[e] = a >> 27;
            const long long ts = tiny[e * 128];
            acc128_add(lv[e], hv[e], (unsigned long long)ts << 17, ts >> 47);
        }
        __syncthreads();  // every thread has read its element-major entries
#pragma unroll
        for (int e = 0; e < VEC; ++e) {  // layout [slot][e][piece]
            red_hi[slot * D + e * CPR + piece] = hv[e];
            red_lo[slot * D + e * CPR + piece] = (long long)lv[e];
        }
    }
    __syncthreads();
    if (t < D) {
        // thread t reduces column piece * VEC + e with piece = t % CPR, e = t / CPR: its
        // slot partials sit at q * D + t in the [slot][e][piece] layout
        const int col = (t % CPR) * VEC + t / CPR;
        long long sh = 0;
        unsigned long long sl = 0;
        for (int q = 0; q < RPI; ++q) acc128_add(sl, sh, (unsigned long long)red_lo[q * D + t], red_hi[q * D + t]);
        // one correct rounding of the exact sum to float64, then the IEEE division by n
        const double mean = ldexp(i128_to_double_rn(sh, sl), -64) / (double)n;
        T* c = C + ((size_t)bh * K + k) * D + col;
        if (sizeof(T) == 2)
            reinterpret_cast<uint16_t*>(c)[0] = double_to_bf16_bits(mean);
        else
            reinterpret_cast<float*>(c)[0] = __double2float_rn(mean);
    }
}

int launch_update(const void* X, int dtype, int BH, int N, int D, int K, const int32_t* perm,
                  const int32_t* offsets, void* C, const int32_t* wide, const uint8_t* tiny_rows,
                  cudaStream_t st) {
    dim3 g(K, BH);
    const int vec = dtype == PARK_BF16 ? 8 : 4;
    if (D % vec || D / vec > 128) return PARK_ERR_UNSUPPORTED;
    const int rpi = 128 / (D / vec);
    ::park::prof_begin(st);
    if (dtype == PARK_BF16)
        k_update<bf16_t><<<g, 128, (size_t)rpi * D * 16, st>>>((const bf16_t*)X, perm, offsets, N, D, K, (bf16_t*)C,
                                                                wide, tiny_rows);
    else
        k_update<float><<<g, 128, (size_t)rpi * D * 16, st>>>((const float*)X, perm, offsets, N, D, K, (float*)C,
                                                               nullptr, nullptr);
    PARK_TRY_LAUNCH("k_update", st);
    return PARK_OK;
}

}  // namespace park
