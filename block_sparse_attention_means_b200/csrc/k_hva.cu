// HyperVAttention's two clustering parts ("HyperVAttention: Efficient Sparse
// Attention with Spatio-Temporal Clustering for Video Diffusion", abstract) on
// this library's K-means and attention:
//
// * 3D local-window K-means.  The video grid is tiled by fixed windows of
//   wt x wh x ww tokens; window w owns centroids floor(w K / nW) ..
//   floor((w+1) K / nW) - 1 and a grid token searches only its window's
//   centroids (text tokens, which have no grid position, search all of them).
//   The assign becomes a stream over X with a handful of candidates per token:
//   float32 scores with a rigorous error bound, float64 for the rows the bound
//   cannot decide.
// * CTA-aligned query-cluster merging.  After the selection, query clusters
//   merge in parallel agglomerative rounds (mutual best partners) whenever the
//   merged cluster needs fewer (query tile, key tile) pairs of the attention
//   kernel than the two apart; a merged cluster keeps the union of its members'
//   kept key clusters.
#include "kernels.h"

namespace park {

namespace {

__device__ inline void window_box(const WinGeom& g, int wi, int& t0, int& y0, int& x0, int& bt, int& by, int& bw) {
    const int c = wi % g.nWw, b = (wi / g.nWw) % g.nWh, a = wi / (g.nWw * g.nWh);
    t0 = a * g.wt;
    y0 = b * g.wh;
    x0 = c * g.ww;
    bt = min(g.wt, g.T - t0);
    by = min(g.wh, g.Hg - y0);
    bw = min(g.ww, g.W - x0);
}

// token index of the l-th member (token order) of the window with origin (t0, y0, x0) and extent (., by, bw)
__device__ inline int window_token(const WinGeom& g, int t0, int y0, int x0, int by, int bw, int l) {
    const int lw = l % bw, ly = (l / bw) % by, lt = l / (bw * by);
    return ((t0 + lt) * g.Hg + (y0 + ly)) * g.W + (x0 + lw);
}

__device__ inline int win_first_centroid(long long wi, int K, int nW) { return (int)(wi * K / nW); }

// 8 consecutive elements as float (exact for both input types)
template <typename T>
__device__ inline void load8(const T* p, float* v);
template <>
__device__ inline void load8<bf16_t>(const bf16_t* p, float* v) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
template <>
__device__ inline void load8<float>(const float* p, float* v) {
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

}  // namespace

// ---------------------------------------------------------------- local init
// Centroid j of window w is the window's member floor(j n_w / K_w) (token order).
template <typename T>
__global__ void k_local_init(const T* __restrict__ X, int N, int D, int K, WinGeom g, T* __restrict__ C) {
    const int k = blockIdx.x, bh = blockIdx.y;
    const int wi = (int)(((long long)(k + 1) * g.nW - 1) / K);
    const int k0 = win_first_centroid(wi, K, g.nW), kw = win_first_centroid(wi + 1, K, g.nW) - k0;
    int t0, y0, x0, bt, by, bw;
    window_box(g, wi, t0, y0, x0, bt, by, bw);
    const int n = bt * by * bw;
    const int l = (int)(((long long)(k - k0) * n) / kw);
    const int tok = window_token(g, t0, y0, x0, by, bw, l);
    const T* src = X + ((size_t)bh * N + tok) * D;
    T* dst = C + ((size_t)bh * K + k) * D;
    for (int j = threadIdx.x; j < D; j += blockDim.x) dst[j] = src[j];
}

// ---------------------------------------------------------------- local assign
// One CTA per (window, 512-token chunk, head); each thread scores two tokens of
// the window against the window's candidates, KC at a time, staged in shared
// memory as float32: s_k = fl32(bias_k) - 2 x . fl32(w_k) with w = c (Euclidean)
// or M c (QRKC).  The float32 winner is certified when the runner-up is more
// than 2 beta above it, with
//   beta = 1.05 (2 u Bmax + (2 D + 7) u ||x|| Wmax),  u = 2^-24,
// which bounds the error of each float32 score against the exact one (the
// roundings of bias and w, the D-term FMA chain, the final subtraction); Wmax and
// Bmax are the head's max ||w_k|| and |bias_k|.  Otherwise the token is
// rescored in float64 (Euclidean sum_j (x_j - c_j)^2; QRKC bias - 2 x . (M c)),
// ties to the lowest index.
constexpr int kLocalThreads = 256;
constexpr int kLocalTokens = 2 * kLocalThreads;

template <typename T, bool METRIC, int KC>
__global__ __launch_bounds__(kLocalThreads) void k_assign_local(
    const T* __restrict__ X, int N, int D, int K, WinGeom g, int chunks, const T* __restrict__ C,
    const double* __restrict__ w64, const double* __restrict__ b64, const float* __restrict__ wmax,
    const float* __restrict__ bmax, int32_t* __restrict__ labels, int64_t* __restrict__ counters, int cnt_slot) {
    extern __shared__ __align__(16) float lsm[];
    __shared__ int s_rescored;
    const int bh = blockIdx.y, wi = blockIdx.x / chunks, ch = blockIdx.x % chunks, tid = threadIdx.x;
    int t0, y0, x0, bt, by, bw;
    window_box(g, wi, t0, y0, x0, bt, by, bw);
    const int n = bt * by * bw;
    if (ch * kLocalTokens >= n) return;  // uniform over the CTA
    const int k0 = win_first_centroid(wi, K, g.nW), kw = win_first_centroid(wi + 1, K, g.nW) - k0;
    const int kpad = (kw + KC - 1) / KC * KC;
    float* wsm = lsm;              // [kpad][D]
    float* bsm = lsm + kpad * D;   // [kpad]
    for (int i = tid; i < kpad * D; i += kLocalThreads) {
        const int j = i / D, d = i - j * D;
        float v = 0.f;
        if (j < kw) {
            const size_t row = (size_t)bh * K + k0 + j;
            v = METRIC ? (float)w64[row * D + d] : Elem<T>::to_float(C + row * D, d);
        }
        wsm[i] = v;
    }
    for (int j = tid; j < kpad; j += kLocalThreads)
        bsm[j] = j < kw ? (float)b64[(size_t)bh * K + k0 + j] : __int_as_float(0x7f800000);
    if (tid == 0) s_rescored = 0;
    __syncthreads();

    const int l0 = ch * kLocalTokens + tid, l1 = l0 + kLocalThreads;
    const bool v0 = l0 < n, v1 = l1 < n;
    const int i0 = window_token(g, t0, y0, x0, by, bw, v0 ? l0 : 0);
    const int i1 = window_token(g, t0, y0, x0, by, bw, v1 ? l1 : 0);
    const T* x0p = X + ((size_t)bh * N + i0) * D;
    const T* x1p = X + ((size_t)bh * N + i1) * D;
    const float INF = __int_as_float(0x7f800000);
    float best0 = INF, sec0 = INF, best1 = INF, sec1 = INF, nx0 = 0.f, nx1 = 0.f;
    int bi0 = 0, bi1 = 0;
    for (int kc = 0; kc < kw; kc += KC) {
        float acc0[KC], acc1[KC];
#pragma unroll
        for (int j = 0; j < KC; ++j) acc0[j] = acc1[j] = 0.f;
        for (int d = 0; d < D; d += 8) {
            float xa[8], xb[8];
            load8<T>(x0p + d, xa);
            load8<T>(x1p + d, xb);
            if (kc == 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    nx0 = fmaf(xa[e], xa[e], nx0);
                    nx1 = fmaf(xb[e], xb[e], nx1);
                }
            }
#pragma unroll
            for (int j = 0; j < KC; ++j) {
                const float4 wa = *reinterpret_cast<const float4*>(wsm + (kc + j) * D + d);
                const float4 wb = *reinterpret_cast<const float4*>(wsm + (kc + j) * D + d + 4);
                acc0[j] = fmaf(xa[0], wa.x, acc0[j]);
                acc0[j] = fmaf(xa[1], wa.y, acc0[j]);
                acc0[j] = fmaf(xa[2], wa.z, acc0[j]);
                acc0[j] = fmaf(xa[3], wa.w, acc0[j]);
                acc0[j] = fmaf(xa[4], wb.x, acc0[j]);
                acc0[j] = fmaf(xa[5], wb.y, acc0[j]);
                acc0[j] = fmaf(xa[6], wb.z, acc0[j]);
                acc0[j] = fmaf(xa[7], wb.w, acc0[j]);
                acc1[j] = fmaf(xb[0], wa.x, acc1[j]);
                acc1[j] = fmaf(xb[1], wa.y, acc1[j]);
                acc1[j] = fmaf(xb[2], wa.z, acc1[j]);
                acc1[j] = fmaf(xb[3], wa.w, acc1[j]);
                acc1[j] = fmaf(xb[4], wb.x, acc1[j]);
                acc1[j] = fmaf(xb[5], wb.y, acc1[j]);
                acc1[j] = fmaf(xb[6], wb.z, acc1[j]);
                acc1[j] = fmaf(xb[7], wb.w, acc1[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < KC; ++j) {
            if (kc + j < kw) {
                const float b = bsm[kc + j];
                const float s0 = fmaf(-2.f, acc0[j], b), s1 = fmaf(-2.f, acc1[j], b);
                if (s0 < best0) {
                    sec0 = best0;
                    best0 = s0;
                    bi0 = kc + j;
                } else if (s0 < sec0) {
                    sec0 = s0;
                }
                if (s1 < best1) {
                    sec1 = best1;
                    best1 = s1;
                    bi1 = kc + j;
                } else if (s1 < sec1) {
                    sec1 = s1;
                }
            }
        }
    }
    const float u = 5.9604645e-8f;  // 2^-24
    const float Wm = wmax[bh], Bm = bmax[bh];
    auto certified = [&](float best, float sec, float nx) {
        const float xn = sqrtf(nx) * 1.001f;  // covers the float32 rounding of ||x||^2
        const float beta = 1.05f * (2.f * u * Bm + (2.f * D + 7.f) * u * xn * Wm);
        return kw == 1 || (sec - best > 2.f * beta);  // false for NaN
    };
    auto rescore = [&](const T* xp) -> int {
        double bd = __longlong_as_double(0x7ff0000000000000ll);
        int bk = 0;
        for (int j = 0; j < kw; ++j) {
            const size_t row = (size_t)bh * K + k0 + j;
            double s = 0.0;
            if (METRIC) {
                for (int d = 0; d < D; ++d) s = __fma_rn(Elem<T>::to_double(xp, d), w64[row * D + d], s);
                s = b64[row] - 2.0 * s;
            } else {
                for (int d = 0; d < D; ++d) {
                    const double e = Elem<T>::to_double(xp, d) - Elem<T>::to_double(C + row * D, d);
                    s = __fma_rn(e, e, s);
                }
            }
            if (s < bd) {
                bd = s;
                bk = j;
            }
        }
        return bk;
    };
    int nres = 0;
    if (v0) {
        int lab = bi0;
        if (!certified(best0, sec0, nx0)) {
            lab = rescore(x0p);
            ++nres;
        }
        labels[(size_t)bh * N + i0] = k0 + lab;
    }
    if (v1) {
        int lab = bi1;
        if (!certified(best1, sec1, nx1)) {
            lab = rescore(x1p);
            ++nres;
        }
        labels[(size_t)bh * N + i1] = k0 + lab;
    }
    if (nres) atomicAdd(&s_rescored, nres);
    __syncthreads();
    if (tid == 0 && s_rescored && counters)
        atomicAdd((unsigned long long*)(counters + cnt_slot), (unsigned long long)s_rescored);
}

int launch_local_init(const void* X, int dtype, int BH, int N, int D, int K, const WinGeom& g, void* C,
                      cudaStream_t st) {
    ::park::prof_begin(st);
    const dim3 grid(K, BH);
    if (dtype == PARK_BF16)
        k_local_init<bf16_t><<<grid, 128, 0, st>>>((const bf16_t*)X, N, D, K, g, (bf16_t*)C);
    else
        k_local_init<float><<<grid, 128, 0, st>>>((const float*)X, N, D, K, g, (float*)C);
    PARK_TRY_LAUNCH("k_local_init", st);
    return PARK_OK;
}

size_t local_assign_smem(int K, int nW, int D) {
    const int kmax = (K + nW - 1) / nW;  // most centroids a window owns
    const int kpad = (kmax + 15) / 16 * 16;
    return (size_t)kpad * (D + 1) * sizeof(float);
}

template <typename T, bool METRIC, int KC>
static void launch_local_kc(dim3 grid, size_t sm, cudaStream_t st, const void* X, int N, int D, int K,
                            const WinGeom& g, int chunks, const void* C, const double* w64, const double* b64,
                            const float* wmax, const float* bmax, int32_t* labels, int64_t* counters, int slot) {
    cudaFuncSetAttribute(k_assign_local<T, METRIC, KC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_assign_local<T, METRIC, KC><<<grid, kLocalThreads, sm, st>>>((const T*)X, N, D, K, g, chunks, (const T*)C,
                                                                   w64, b64, wmax, bmax, labels, counters, slot);
}

template <typename T, bool METRIC>
static void launch_local_t(dim3 grid, size_t sm, int kmax, cudaStream_t st, const void* X, int N, int D, int K,
                           const WinGeom& g, int chunks, const void* C, const double* w64, const double* b64,
                           const float* wmax, const float* bmax, int32_t* labels, int64_t* counters, int slot) {
    if (kmax <= 4)
        launch_local_kc<T, METRIC, 4>(grid, sm, st, X, N, D, K, g, chunks, C, w64, b64, wmax, bmax, labels, counters,
                                      slot);
    else if (kmax <= 8)
        launch_local_kc<T, METRIC, 8>(grid, sm, st, X, N, D, K, g, chunks, C, w64, b64, wmax, bmax, labels, counters,
                                      slot);
    else
        launch_local_kc<T, METRIC, 16>(grid, sm, st, X, N, D, K, g, chunks, C, w64, b64, wmax, bmax, labels,
                                       counters, slot);
}

int launch_assign_local(const void* X, int dtype, int BH, int N, int D, int K, const WinGeom& g, const void* C,
                        const double* w64, const double* b64, const float* wmax, const float* bmax, int32_t* labels,
                        int64_t* counters, int cnt_slot, cudaStream_t st) {
    if (D % 8 != 0 || D > 128) return PARK_ERR_UNSUPPORTED;
    const int chunks = (g.maxwin + kLocalTokens - 1) / kLocalTokens;
    const dim3 grid(g.nW * chunks, BH);
    const size_t sm = local_assign_smem(K, g.nW, D);
    const int kmax = (K + g.nW - 1) / g.nW;
    const bool metric = w64 != nullptr;
    ::park::prof_begin(st);
    if (dtype == PARK_BF16) {
        if (metric)
            launch_local_t<bf16_t, true>(grid, sm, kmax, st, X, N, D, K, g, chunks, C, w64, b64, wmax, bmax, labels,
                                         counters, cnt_slot);
        else
            launch_local_t<bf16_t, false>(grid, sm, kmax, st, X, N, D, K, g, chunks, C, w64, b64, wmax, bmax, labels,
                                          counters, cnt_slot);
    } else {
        if (metric)
            launch_local_t<float, true>(grid, sm, kmax, st, X, N, D, K, g, chunks, C, w64, b64, wmax, bmax, labels,
                                        counters, cnt_slot);
        else
            launch_local_t<float, false>(grid, sm, kmax, st, X, N, D, K, g, chunks, C, w64, b64, wmax, bmax, labels,
                                         counters, cnt_slot);
    }
    PARK_TRY_LAUNCH("k_assign_local", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- cluster merging
// Per head: S[r] = bitset of query cluster r's kept key clusters (Wd words),
// n[r] its rows, L[r] the padded key rows of S[r] in 8-row units, and the key
// clusters' unit counts wk[m] held as bit planes P[b] (m in P[b] when bit b of
// wk[m] is set), so the units kept by both g and h are
//   sum_b 2^b popc(S[g] & S[h] & P[b]).
// cost(n, L) = ceil(n / 128) * ceil(L / 16): the attention's (query tile, key
// tile) pairs for the group.
namespace {

__device__ inline int merge_cost(int n, int L) { return ((n + 127) >> 7) * ((L + 15) >> 4); }

}  // namespace

__global__ void k_merge_init(const uint8_t* __restrict__ mask, const int32_t* __restrict__ q_off,
                             const int32_t* __restrict__ k_off, int NQ, int NK, int Wd, MergeWs m) {
    const int r = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const uint8_t* row = mask + ((size_t)bh * NQ + r) * NK;
    const int32_t* ko = k_off + (size_t)bh * (NK + 1);
    uint32_t* S = m.S + ((size_t)bh * NQ + r) * Wd;
    int L = 0;
    for (int w = tid; w < Wd; w += blockDim.x) {
        uint32_t bits = 0;
        for (int b = 0; b < 32; ++b) {
            const int k = 32 * w + b;
            if (k < NK && row[k]) {
                bits |= 1u << b;
                L += (ko[k + 1] - ko[k] + 7) >> 3;
            }
        }
        S[w] = bits;
    }
    L = warp_sum_int(L);
    __shared__ int red[32];
    if ((tid & 31) == 0) red[tid >> 5] = L;
    __syncthreads();
    if (tid == 0) {
        int t = 0;
        for (int q = 0; q < (int)(blockDim.x >> 5); ++q) t += red[q];
        const size_t i = (size_t)bh * NQ + r;
        const int n = q_off[(size_t)bh * (NQ + 1) + r + 1] - q_off[(size_t)bh * (NQ + 1) + r];
        m.n[i] = n;
        m.L[i] = t;
        m.alive[i] = n > 0;
        m.root[i] = r;
        m.best[i] = -1;
    }
}

__global__ void k_merge_planes(const int32_t* __restrict__ k_off, int NQ, int NK, int Wd, MergeWs m) {
    const int bh = blockIdx.x, tid = threadIdx.x;
    const int32_t* ko = k_off + (size_t)bh * (NK + 1);
    __shared__ int s_max;
    if (tid == 0) {
        s_max = 0;
        m.done[bh] = 0;
    }
    __syncthreads();
    for (int w = tid; w < Wd; w += blockDim.x) {
        uint32_t planes[kMergePlanes];
#pragma unroll
        for (int b = 0; b < kMergePlanes; ++b) planes[b] = 0;
        int mx = 0;
        for (int q = 0; q < 32; ++q) {
            const int k = 32 * w + q;
            if (k >= NK) break;
            const int u = (ko[k + 1] - ko[k] + 7) >> 3;
            mx = max(mx, u);
#pragma unroll
            for (int b = 0; b < kMergePlanes; ++b)
                if ((u >> b) & 1) planes[b] |= 1u << q;
        }
#pragma unroll
        for (int b = 0; b < kMergePlanes; ++b) m.P[((size_t)bh * kMergePlanes + b) * Wd + w] = planes[b];
        atomicMax(&s_max, mx);
    }
    __syncthreads();
    if (tid == 0) m.nb[bh] = 32 - __clz(s_max);
}

// One CTA per 8 groups g of a head: the best partner h of each (largest positive
// gain, ties to the lowest h), -1 when no merge gains.  A pair is skipped
// without counting when even a union adding no key rows could not gain:
// ceil((n_g + n_h)/128) * max(T_g, T_h) >= cost_g + cost_h.
constexpr int kMergeGroups = 8;

__global__ __launch_bounds__(256) void k_merge_best(int NQ, int Wd, MergeWs m) {
    extern __shared__ uint32_t gp[];  // [kMergeGroups][nb][Wd]: S[g] & P[b]
    __shared__ int sg_n[kMergeGroups], sg_L[kMergeGroups], sg_cost[kMergeGroups], sg_T[kMergeGroups];
    __shared__ int red_gain[8][kMergeGroups], red_h[8][kMergeGroups];
    const int bh = blockIdx.y, g0 = blockIdx.x * kMergeGroups, tid = threadIdx.x;
    if (m.done[bh]) return;
    const int nb = m.nb[bh];
    const size_t hb = (size_t)bh * NQ;
    if (tid < kMergeGroups) {
        const int g = g0 + tid;
        const bool ok = g < NQ && m.alive[hb + g];
        sg_n[tid] = ok ? m.n[hb + g] : 0;
        sg_L[tid] = ok ? m.L[hb + g] : 0;
        sg_cost[tid] = ok ? merge_cost(sg_n[tid], sg_L[tid]) : -1;
        sg_T[tid] = ok ? (sg_L[tid] + 15) >> 4 : 0;
    }
    for (int i = tid; i < kMergeGroups * nb * Wd; i += blockDim.x) {
        const int q = i / (nb * Wd), rem = i - q * nb * Wd, b = rem / Wd, w = rem - b * Wd;
        const int g = g0 + q;
        gp[i] = g < NQ ? m.S[(hb + g) * Wd + w] & m.P[((size_t)bh * kMergePlanes + b) * Wd + w] : 0u;
    }
    __syncthreads();
    int bgain[kMergeGroups], bh_idx[kMergeGroups];
#pragma unroll
    for (int q = 0; q < kMergeGroups; ++q) {
        bgain[q] = 0;
        bh_idx[q] = -1;
    }
    for (int h = tid; h < NQ; h += blockDim.x) {
        if (!m.alive[hb + h]) continue;
        const int nh = m.n[hb + h], Lh = m.L[hb + h];
        const int Th = (Lh + 15) >> 4, ch = merge_cost(nh, Lh);
        unsigned need = 0;
#pragma unroll
        for (int q = 0; q < kMergeGroups; ++q) {
            if (sg_cost[q] >= 0 && g0 + q != h) {
                const int A = (sg_n[q] + nh + 127) >> 7;
                if (A * max(sg_T[q], Th) < sg_cost[q] + ch) need |= 1u << q;
            }
        }
        if (!need) continue;
        int inter[kMergeGroups];
#pragma unroll
        for (int q = 0; q < kMergeGroups; ++q) inter[q] = 0;
        const uint32_t* Sh = m.S + (hb + h) * Wd;
        for (int w = 0; w < Wd; ++w) {
            const uint32_t s = Sh[w];
            if (!s) continue;
#pragma unroll
            for (int q = 0; q < kMergeGroups; ++q) {
                if ((need >> q) & 1u) {
                    const uint32_t* gq = gp + (size_t)q * nb * Wd + w;
                    int acc = 0;
                    for (int b = 0; b < nb; ++b) acc += __popc(s & gq[b * Wd]) << b;
                    inter[q] += acc;
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kMergeGroups; ++q) {
            if ((need >> q) & 1u) {
                const int Lu = sg_L[q] + Lh - inter[q];
                const int gain = sg_cost[q] + ch - merge_cost(sg_n[q] + nh, Lu);
                if (gain > bgain[q]) {  // h ascends within a thread: strict keeps the lowest
                    bgain[q] = gain;
                    bh_idx[q] = h;
                }
            }
        }
    }
    // block argmax per group: largest gain, then lowest h
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int q = 0; q < kMergeGroups; ++q) {
        int gq = bgain[q], hq = bh_idx[q];
        for (int o = 16; o > 0; o >>= 1) {
            const int go = __shfl_xor_sync(0xffffffffu, gq, o), ho = __shfl_xor_sync(0xffffffffu, hq, o);
            if (go > gq || (go == gq && ho >= 0 && (hq < 0 || ho < hq))) {
                gq = go;
                hq = ho;
            }
        }
        if (lane == 0) {
            red_gain[warp][q] = gq;
            red_h[warp][q] = hq;
        }
    }
    __syncthreads();
    if (tid < kMergeGroups && g0 + tid < NQ) {
        int gq = 0, hq = -1;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            const int go = red_gain[w][tid], ho = red_h[w][tid];
            if (go > gq || (go == gq && ho >= 0 && (hq < 0 || ho < hq))) {
                gq = go;
                hq = ho;
            }
        }
        m.best[hb + g0 + tid] = gq > 0 ? hq : -1;
    }
}

// Mutual best pairs merge into the lower index; a head with no merge is done.
__global__ void k_merge_apply(int NQ, int Wd, MergeWs m) {
    const int bh = blockIdx.x, tid = threadIdx.x;
    if (m.done[bh]) return;
    __shared__ int any;
    if (tid == 0) any = 0;
    __syncthreads();
    const size_t hb = (size_t)bh * NQ;
    const int nb = m.nb[bh];
    for (int g = tid; g < NQ; g += blockDim.x) {
        const int h = m.best[hb + g];
        if (h > g && m.best[hb + h] == g) {
            uint32_t* Sg = m.S + (hb + g) * Wd;
            uint32_t* Sh = m.S + (hb + h) * Wd;
            int L = 0;
            for (int w = 0; w < Wd; ++w) {
                const uint32_t s = Sg[w] | Sh[w];
                Sg[w] = s;
                Sh[w] = 0u;
                for (int b = 0; b < nb; ++b) L += __popc(s & m.P[((size_t)bh * kMergePlanes + b) * Wd + w]) << b;
            }
            m.L[hb + g] = L;
            m.L[hb + h] = 0;
            m.n[hb + g] += m.n[hb + h];
            m.n[hb + h] = 0;
            m.alive[hb + h] = 0;
            m.root[hb + h] = g;
            any = 1;
        }
    }
    __syncthreads();
    if (tid == 0 && !any) m.done[bh] = 1;
}

// Final groups: every cluster's root; a live root's mask row becomes its union,
// a merged-away row is cleared; kept counts follow.
__global__ void k_merge_finalize(int NQ, int NK, int Wd, MergeWs m, uint8_t* __restrict__ mask,
                                 int32_t* __restrict__ kept_cnt) {
    const int r = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const size_t hb = (size_t)bh * NQ;
    int g = r;
    for (int hop = 0; hop < NQ && m.root[hb + g] != g; ++hop) g = m.root[hb + g];
    if (tid == 0) m.rootf[hb + r] = g;
    uint8_t* row = mask + (hb + r) * NK;
    if (g == r && !m.alive[hb + r]) return;  // an empty cluster keeps its (empty) row
    const uint32_t* S = m.S + (hb + r) * Wd;
    const bool keep = g == r;
    for (int k = tid; k < NK; k += blockDim.x) row[k] = keep ? (uint8_t)((S[k >> 5] >> (k & 31)) & 1u) : (uint8_t)0;
    if (tid == 0) {
        int c = 0;
        if (keep)
            for (int w = 0; w < Wd; ++w) c += __popc(S[w]);
        kept_cnt[hb + r] = c;
    }
}

__global__ void k_merge_relabel(int BH, int N, int NQ, const int32_t* __restrict__ rootf, int32_t* __restrict__ labels) {
    const size_t total = (size_t)BH * N;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t bh = i / N;
        labels[i] = rootf[bh * NQ + labels[i]];
    }
}

int launch_merge(uint8_t* mask, int32_t* kept_cnt, const int32_t* q_off, const int32_t* k_off, int BH, int N, int NQ,
                 int NK, int rounds, const MergeWs& m, int32_t* q_labels, int num_sms, cudaStream_t st) {
    const int Wd = (NK + 31) / 32;
    ::park::prof_begin(st);
    k_merge_init<<<dim3(NQ, BH), 128, 0, st>>>(mask, q_off, k_off, NQ, NK, Wd, m);
    PARK_TRY_LAUNCH("k_merge_init", st);
    ::park::prof_begin(st);
    k_merge_planes<<<BH, 128, 0, st>>>(k_off, NQ, NK, Wd, m);
    PARK_TRY_LAUNCH("k_merge_planes", st);
    const size_t sm = (size_t)kMergeGroups * kMergePlanes * Wd * 4;
    if (cudaFuncSetAttribute(k_merge_best, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess) {
        cudaGetLastError();
        return PARK_ERR_CUDA;
    }
    for (int it = 0; it < rounds; ++it) {
        ::park::prof_begin(st);
        k_merge_best<<<dim3((NQ + kMergeGroups - 1) / kMergeGroups, BH), 256, sm, st>>>(NQ, Wd, m);
        PARK_TRY_LAUNCH("k_merge_best", st);
        ::park::prof_begin(st);
        k_merge_apply<<<BH, 1024, 0, st>>>(NQ, Wd, m);
        PARK_TRY_LAUNCH("k_merge_apply", st);
    }
    ::park::prof_begin(st);
    k_merge_finalize<<<dim3(NQ, BH), 128, 0, st>>>(NQ, NK, Wd, m, mask, kept_cnt);
    PARK_TRY_LAUNCH("k_merge_finalize", st);
    ::park::prof_begin(st);
    k_merge_relabel<<<num_sms * 8, 256, 0, st>>>(BH, N, NQ, m.rootf, q_labels);
    PARK_TRY_LAUNCH("k_merge_relabel", st);
    return PARK_OK;
}

}  // namespace park
