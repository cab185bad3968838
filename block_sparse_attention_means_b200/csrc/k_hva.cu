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

// acc0[j] += x_a . w_j and acc1[j] += x_b . w_j (float32 FMA chains over the D
// columns in order) for the KC rows w_j of wsm; the token rows are read 16
// columns at a time, whole 32-byte sectors, so no sector is fetched twice.  With
// NORM the squared norms of the two rows are accumulated too.
template <typename T, int KC, bool NORM>
__device__ inline void dot_rows(const T* xa_p, const T* xb_p, const float* wsm, int D, float* acc0, float* acc1,
                                float& nxa, float& nxb) {
    for (int d = 0; d < D; d += 16) {
        float xa[16], xb[16];
        load8<T>(xa_p + d, xa);
        load8<T>(xa_p + d + 8, xa + 8);
        load8<T>(xb_p + d, xb);
        load8<T>(xb_p + d + 8, xb + 8);
        if (NORM) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                nxa = fmaf(xa[e], xa[e], nxa);
                nxb = fmaf(xb[e], xb[e], nxb);
            }
        }
#pragma unroll
        for (int j = 0; j < KC; ++j) {
#pragma unroll
            for (int h = 0; h < 16; h += 4) {
                const float4 w = *reinterpret_cast<const float4*>(wsm + j * D + d + h);
                acc0[j] = fmaf(xa[h], w.x, acc0[j]);
                acc0[j] = fmaf(xa[h + 1], w.y, acc0[j]);
                acc0[j] = fmaf(xa[h + 2], w.z, acc0[j]);
                acc0[j] = fmaf(xa[h + 3], w.w, acc0[j]);
                acc1[j] = fmaf(xb[h], w.x, acc1[j]);
                acc1[j] = fmaf(xb[h + 1], w.y, acc1[j]);
                acc1[j] = fmaf(xb[h + 2], w.z, acc1[j]);
                acc1[j] = fmaf(xb[h + 3], w.w, acc1[j]);
            }
        }
    }
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
//   beta = 1.05 (2 u Bmax + (2 D + 7) u ||x|| Wmax) + 2^-120 (||x|| + 1),  u = 2^-24,
// which bounds the error of each float32 score against the exact one (the
// roundings of bias and w, the D-term FMA chain, the final subtraction, and
// gradual underflow below 2^-126); Wmax and Bmax are the head's max ||w_k|| and
// |bias_k|.  Otherwise the token is
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
        if (kc == 0)
            dot_rows<T, KC, true>(x0p, x1p, wsm + kc * D, D, acc0, acc1, nx0, nx1);
        else
            dot_rows<T, KC, false>(x0p, x1p, wsm + kc * D, D, acc0, acc1, nx0, nx1);
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
        // + absolute terms for results below the float32 normal range (gradual
        // underflow: <= 2^-150 per rounding, generously covered)
        const float beta = 1.05f * (2.f * u * Bm + (2.f * D + 7.f) * u * xn * Wm) + xn * 0x1p-120f + 0x1p-120f;
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

// ---------------------------------------------------------------- text tokens
// Text tokens have no box and search every centroid.  k_text_partial: one CTA
// per (64 text tokens, split of the centroids, head); lane l holds tokens l and
// l + 32, warp w scores candidates 16w .. 16w + 15 of each staged block of 128
// centroids (float32 operands in shared memory, the same scores as the box
// assign) and the CTA leaves each token's (best, index, runner-up) of its split.
// k_text_finish: one warp per token merges the splits, certifies the winner with
// the box assign's bound, else rescores it in float64 (lanes over the columns,
// one centroid at a time, ties to the lowest index).
constexpr int kTextTokens = 64;
constexpr int kTextBlock = 128;

int text_splits(int BH, int n_text, int K) {
    const int nblk = (K + kTextBlock - 1) / kTextBlock;
    const long long ctas = (long long)BH * ((n_text + kTextTokens - 1) / kTextTokens);
    long long want = (4 * 148 + ctas - 1) / ctas;  // about four CTAs per SM of a B200
    if (want < 1) want = 1;
    const int bps = (int)((nblk + want - 1) / want);  // centroid blocks per split
    return (nblk + bps - 1) / bps;
}

struct TextPart {
    float best, sec;
    int idx, pad;
};

template <typename T, bool METRIC>
__global__ __launch_bounds__(256) void k_text_partial(const T* __restrict__ X, int N, int D, int K, int row0,
                                                      int splits, const T* __restrict__ C,
                                                      const double* __restrict__ w64, const double* __restrict__ b64,
                                                      TextPart* __restrict__ part) {
    extern __shared__ __align__(16) float tsm[];
    float* wsm = tsm;                        // [kTextBlock][D]
    float* bsm = tsm + kTextBlock * D;       // [kTextBlock]
    __shared__ float r_best[8][kTextTokens], r_sec[8][kTextTokens];
    __shared__ int r_idx[8][kTextTokens];
    const int bh = blockIdx.z, sp = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_text = N - row0;
    const int nblk = (K + kTextBlock - 1) / kTextBlock, bps = (nblk + splits - 1) / splits;
    const int kb = sp * bps * kTextBlock, ke = min(K, (sp + 1) * bps * kTextBlock);
    const int ta = blockIdx.x * kTextTokens + lane, tb = ta + 32;
    const T* xa_p = X + ((size_t)bh * N + row0 + min(ta, n_text - 1)) * D;
    const T* xb_p = X + ((size_t)bh * N + row0 + min(tb, n_text - 1)) * D;
    const float INF = __int_as_float(0x7f800000);
    float best0 = INF, sec0 = INF, best1 = INF, sec1 = INF;
    int bi0 = kb, bi1 = kb;
    for (int cb = kb; cb < ke; cb += kTextBlock) {
        __syncthreads();  // the previous block is consumed
        const int nb = min(kTextBlock, ke - cb);
        for (int i = tid; i < kTextBlock * D; i += blockDim.x) {
            const int j = i / D, d = i - j * D;
            float v = 0.f;
            if (j < nb) {
                const size_t row = (size_t)bh * K + cb + j;
                v = METRIC ? (float)w64[row * D + d] : Elem<T>::to_float(C + row * D, d);
            }
            wsm[i] = v;
        }
        for (int j = tid; j < kTextBlock; j += blockDim.x) bsm[j] = j < nb ? (float)b64[(size_t)bh * K + cb + j] : INF;
        __syncthreads();
        const int c0 = 16 * warp;
        if (c0 >= nb) continue;
        float acc0[16], acc1[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) acc0[j] = acc1[j] = 0.f;
        float na = 0.f, nb2 = 0.f;
        dot_rows<T, 16, false>(xa_p, xb_p, wsm + c0 * D, D, acc0, acc1, na, nb2);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (c0 + j < nb) {
                const float b = bsm[c0 + j];
                const float s0 = fmaf(-2.f, acc0[j], b), s1 = fmaf(-2.f, acc1[j], b);
                const int k = cb + c0 + j;
                if (s0 < best0) {
                    sec0 = best0;
                    best0 = s0;
                    bi0 = k;
                } else if (s0 < sec0) {
                    sec0 = s0;
                }
                if (s1 < best1) {
                    sec1 = best1;
                    best1 = s1;
                    bi1 = k;
                } else if (s1 < sec1) {
                    sec1 = s1;
                }
            }
        }
    }
    r_best[warp][lane] = best0;
    r_sec[warp][lane] = sec0;
    r_idx[warp][lane] = bi0;
    r_best[warp][lane + 32] = best1;
    r_sec[warp][lane + 32] = sec1;
    r_idx[warp][lane + 32] = bi1;
    __syncthreads();
    if (tid < kTextTokens) {
        const int t = blockIdx.x * kTextTokens + tid;
        int ww = 0;  // winner over the warps (ties: lowest index), runner-up over the rest
        for (int w = 1; w < 8; ++w)
            if (r_best[w][tid] < r_best[ww][tid] || (r_best[w][tid] == r_best[ww][tid] && r_idx[w][tid] < r_idx[ww][tid]))
                ww = w;
        float sec = r_sec[ww][tid];
        for (int w = 0; w < 8; ++w)
            if (w != ww) sec = fminf(sec, r_best[w][tid]);
        if (t < n_text) part[((size_t)bh * n_text + t) * splits + sp] = TextPart{r_best[ww][tid], sec, r_idx[ww][tid], 0};
    }
}

template <typename T, bool METRIC>
__global__ __launch_bounds__(256) void k_text_finish(const T* __restrict__ X, int N, int D, int K, int row0,
                                                     int splits, const T* __restrict__ C,
                                                     const double* __restrict__ w64, const double* __restrict__ b64,
                                                     const float* __restrict__ wmax, const float* __restrict__ bmax,
                                                     const TextPart* __restrict__ part, int32_t* __restrict__ labels,
                                                     int64_t* __restrict__ counters, int cnt_slot) {
    __shared__ int s_list[8], s_n;
    __shared__ double s_x[128];
    __shared__ double s_bd[8];
    __shared__ int s_bk[8];
    const int bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_text = N - row0;
    const int t = blockIdx.x * 8 + warp;
    if (tid == 0) s_n = 0;
    __syncthreads();
    if (t < n_text) {  // warp-uniform
        const float INF = __int_as_float(0x7f800000);
        float best = INF, sec = INF;
        int idx = K;
        if (lane < splits) {
            const TextPart pp = part[((size_t)bh * n_text + t) * splits + lane];
            best = pp.best;
            sec = pp.sec;
            idx = pp.idx;
        }
        for (int o = 16; o > 0; o >>= 1) {  // merge (best, idx, sec) over the splits
            const float ob = __shfl_xor_sync(0xffffffffu, best, o), os = __shfl_xor_sync(0xffffffffu, sec, o);
            const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
            if (ob < best || (ob == best && oi < idx)) {
                sec = fminf(best, os);
                best = ob;
                idx = oi;
            } else {
                sec = fminf(sec, ob);
            }
        }
        const T* xp = X + ((size_t)bh * N + row0 + t) * D;
        float nx = 0.f;
        for (int j = lane; j < D; j += 32) {
            const float v = Elem<T>::to_float(xp, j);
            nx = fmaf(v, v, nx);
        }
        nx = warp_sum(nx);
        const float u = 5.9604645e-8f;  // 2^-24
        const float xn = sqrtf(nx) * 1.001f;
        const float beta = 1.05f * (2.f * u * bmax[bh] + (2.f * D + 7.f) * u * xn * wmax[bh]) + xn * 0x1p-120f +
                           0x1p-120f;
        if (lane == 0) {
            if (K == 1 || sec - best > 2.f * beta)
                labels[(size_t)bh * N + row0 + t] = idx < K ? idx : 0;
            else
                s_list[atomicAdd(&s_n, 1)] = t;
        }
    }
    __syncthreads();
    // float64 rescore of the undecided tokens with the whole CTA: thread i scores
    // centroids i, i + 256, ... (ascending), then a CTA argmin, ties to the lowest index
    const int nlist = s_n;
    for (int e = 0; e < nlist; ++e) {
        const int tt = s_list[e];
        const T* xp = X + ((size_t)bh * N + row0 + tt) * D;
        for (int j = tid; j < D; j += blockDim.x) s_x[j] = Elem<T>::to_double(xp, j);
        __syncthreads();
        double bd = __longlong_as_double(0x7ff0000000000000ll);
        int bk = 0;
        for (int k = tid; k < K; k += blockDim.x) {
            const size_t row = (size_t)bh * K + k;
            double sc = 0.0;
            if (METRIC) {
                const double* wr = w64 + row * D;
                for (int d = 0; d < D; ++d) sc = __fma_rn(s_x[d], wr[d], sc);
                sc = b64[row] - 2.0 * sc;
            } else {
                const T* cr = C + row * D;
                for (int d = 0; d < D; ++d) {
                    const double df = s_x[d] - Elem<T>::to_double(cr, d);
                    sc = __fma_rn(df, df, sc);
                }
            }
            if (sc < bd) {
                bd = sc;
                bk = k;
            }
        }
        for (int o = 16; o > 0; o >>= 1) {
            const double od = __shfl_xor_sync(0xffffffffu, bd, o);
            const int ok = __shfl_xor_sync(0xffffffffu, bk, o);
            if (od < bd || (od == bd && ok < bk)) {
                bd = od;
                bk = ok;
            }
        }
        if (lane == 0) {
            s_bd[warp] = bd;
            s_bk[warp] = bk;
        }
        __syncthreads();
        if (tid == 0) {
            for (int w = 1; w < 8; ++w)
                if (s_bd[w] < bd || (s_bd[w] == bd && s_bk[w] < bk)) {
                    bd = s_bd[w];
                    bk = s_bk[w];
                }
            labels[(size_t)bh * N + row0 + tt] = bk;
        }
        __syncthreads();
    }
    if (tid == 0 && nlist && counters)
        atomicAdd((unsigned long long*)(counters + cnt_slot), (unsigned long long)nlist);
}

// enough for any K' <= K (the split count is not monotone in K)
size_t text_scratch_bytes(int BH, int n_text, int K) {
    if (n_text <= 0) return 0;
    int most = 1;
    for (int k = 1; k <= K; k += kTextBlock) most = max(most, text_splits(BH, n_text, k));
    most = max(most, text_splits(BH, n_text, K));
    return (size_t)BH * n_text * most * sizeof(TextPart);
}

int launch_assign_text(const void* X, int dtype, int BH, int N, int D, int K, int row0, const void* C,
                       const double* w64, const double* b64, const float* wmax, const float* bmax, void* scratch,
                       int32_t* labels, int64_t* counters, int cnt_slot, cudaStream_t st) {
    if (D % 16 != 0 || D > 128) return PARK_ERR_UNSUPPORTED;
    const int n_text = N - row0;
    if (n_text <= 0) return PARK_OK;
    const int splits = text_splits(BH, n_text, K);
    const dim3 g1((n_text + kTextTokens - 1) / kTextTokens, splits, BH), g2((n_text + 7) / 8, BH);
    const size_t sm = (size_t)kTextBlock * (D + 1) * sizeof(float);
    TextPart* part = static_cast<TextPart*>(scratch);
    const bool metric = w64 != nullptr;
#define PARK_TEXT_LAUNCH(T, M)                                                                                     \
    do {                                                                                                           \
        cudaFuncSetAttribute(k_text_partial<T, M>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);         \
        ::park::prof_begin(st);                                                                                    \
        k_text_partial<T, M><<<g1, 256, sm, st>>>((const T*)X, N, D, K, row0, splits, (const T*)C, w64, b64, part); \
        PARK_TRY_LAUNCH("k_text_partial", st);                                                                     \
        ::park::prof_begin(st);                                                                                    \
        k_text_finish<T, M><<<g2, 256, 0, st>>>((const T*)X, N, D, K, row0, splits, (const T*)C, w64, b64, wmax,   \
                                                bmax, part, labels, counters, cnt_slot);                            \
        PARK_TRY_LAUNCH("k_text_finish", st);                                                                      \
    } while (0)
    if (dtype == PARK_BF16) {
        if (metric) PARK_TEXT_LAUNCH(bf16_t, true);
        else PARK_TEXT_LAUNCH(bf16_t, false);
    } else {
        if (metric) PARK_TEXT_LAUNCH(float, true);
        else PARK_TEXT_LAUNCH(float, false);
    }
#undef PARK_TEXT_LAUNCH
    return PARK_OK;
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
    if (D % 16 != 0 || D > 128) return PARK_ERR_UNSUPPORTED;
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

// Kept units shared by groups g and h, I[g][h] = sum_b 2^b popc(S[g] & S[h] & P[b])
// (symmetric), for the groups flagged in todo (first round: every live group,
// each pair once from its lower index).  A pair that cannot gain whatever it
// shares is stored as -1 without counting: ceil((n_g + n_h)/128) * max(T_g, T_h)
// >= cost_g + cost_h, since the union keeps at least as many key tiles as
// either group.  That test depends only on the two groups, so it stays true
// until one of them merges, which puts it back in todo.
constexpr int kMergeGroups = 8;

__global__ __launch_bounds__(256) void k_merge_inter(int NQ, int Wd, int first, MergeWs m) {
    extern __shared__ uint32_t gp[];  // [kMergeGroups][nb][Wd]: S[g] & P[b]
    __shared__ int sg_n[kMergeGroups], sg_L[kMergeGroups], sg_cost[kMergeGroups], sg_T[kMergeGroups];
    __shared__ int s_any;
    const int bh = blockIdx.y, g0 = blockIdx.x * kMergeGroups, tid = threadIdx.x;
    if (m.done[bh]) return;
    const int nb = m.nb[bh];
    const size_t hb = (size_t)bh * NQ;
    if (tid == 0) s_any = 0;
    __syncthreads();
    if (tid < kMergeGroups) {
        const int g = g0 + tid;
        const bool ok = g < NQ && m.alive[hb + g] && (first || m.todo[hb + g]);
        sg_n[tid] = ok ? m.n[hb + g] : 0;
        sg_L[tid] = ok ? m.L[hb + g] : 0;
        sg_cost[tid] = ok ? merge_cost(sg_n[tid], sg_L[tid]) : -1;
        sg_T[tid] = ok ? (sg_L[tid] + 15) >> 4 : 0;
        if (ok) atomicOr(&s_any, 1);
    }
    __syncthreads();
    if (!s_any) return;  // uniform
    for (int i = tid; i < kMergeGroups * nb * Wd; i += blockDim.x) {
        const int q = i / (nb * Wd), rem = i - q * nb * Wd, b = rem / Wd, w = rem - b * Wd;
        const int g = g0 + q;
        gp[i] = (g < NQ && sg_cost[q] >= 0) ? m.S[(hb + g) * Wd + w] & m.P[((size_t)bh * kMergePlanes + b) * Wd + w]
                                             : 0u;
    }
    __syncthreads();
    int32_t* I = m.inter + hb * NQ;
    for (int h = tid; h < NQ; h += blockDim.x) {
        if (!m.alive[hb + h]) continue;
        const int nh = m.n[hb + h], Lh = m.L[hb + h];
        const int Th = (Lh + 15) >> 4, ch = merge_cost(nh, Lh);
        unsigned want = 0, need = 0;
#pragma unroll
        for (int q = 0; q < kMergeGroups; ++q) {
            const int g = g0 + q;
            if (sg_cost[q] >= 0 && g != h && (!first || h > g)) {
                want |= 1u << q;
                const int A = (sg_n[q] + nh + 127) >> 7;
                if (A * max(sg_T[q], Th) < sg_cost[q] + ch) need |= 1u << q;
            }
        }
        if (!want) continue;
        int inter[kMergeGroups];
#pragma unroll
        for (int q = 0; q < kMergeGroups; ++q) inter[q] = 0;
        if (need) {
            const uint32_t* Sh = m.S + (hb + h) * Wd;
            for (int w = 0; w < Wd; ++w) {
                const uint32_t sw = Sh[w];
                if (!sw) continue;
#pragma unroll
                for (int q = 0; q < kMergeGroups; ++q) {
                    if ((need >> q) & 1u) {
                        const uint32_t* gq = gp + (size_t)q * nb * Wd + w;
                        int acc = 0;
                        for (int b = 0; b < nb; ++b) acc += __popc(sw & gq[b * Wd]) << b;
                        inter[q] += acc;
                    }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kMergeGroups; ++q) {
            if ((want >> q) & 1u) {
                const int g = g0 + q;
                const int v = ((need >> q) & 1u) ? inter[q] : -1;
                I[(size_t)g * NQ + h] = v;
                I[(size_t)h * NQ + g] = v;
            }
        }
    }
}

// One warp per group g: the partner h with the largest gain
// cost(g) + cost(h) - cost(g u h) > 0, ties to the lowest h; -1 if none.
__global__ __launch_bounds__(256) void k_merge_pick(int NQ, MergeWs m) {
    const int bh = blockIdx.y, lane = threadIdx.x & 31;
    const int g = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (m.done[bh] || g >= NQ) return;  // warp-uniform
    const size_t hb = (size_t)bh * NQ;
    if (!m.alive[hb + g]) {
        if (lane == 0) m.best[hb + g] = -1;
        return;
    }
    const int ng = m.n[hb + g], Lg = m.L[hb + g], cg = merge_cost(ng, Lg);
    const int32_t* I = m.inter + (hb + g) * NQ;
    int bgain = 0, bidx = -1;
    for (int h = lane; h < NQ; h += 32) {
        if (h == g || !m.alive[hb + h]) continue;
        const int it = I[h];
        if (it < 0) continue;
        const int nh = m.n[hb + h], Lh = m.L[hb + h];
        const int gain = cg + merge_cost(nh, Lh) - merge_cost(ng + nh, Lg + Lh - it);
        if (gain > bgain) {  // h ascends within a lane: strict keeps the lowest
            bgain = gain;
            bidx = h;
        }
    }
    for (int o = 16; o > 0; o >>= 1) {
        const int go = __shfl_xor_sync(0xffffffffu, bgain, o), ho = __shfl_xor_sync(0xffffffffu, bidx, o);
        if (go > bgain || (go == bgain && ho >= 0 && (bidx < 0 || ho < bidx))) {
            bgain = go;
            bidx = ho;
        }
    }
    if (lane == 0) m.best[hb + g] = bgain > 0 ? bidx : -1;
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
        const bool merge = h > g && m.best[hb + h] == g;
        m.todo[hb + g] = merge;
        if (merge) {
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

int launch_merge_setup(const uint8_t* mask, const int32_t* q_off, const int32_t* k_off, int BH, int NQ, int NK,
                       const MergeWs& m, cudaStream_t st) {
    const int Wd = (NK + 31) / 32;
    ::park::prof_begin(st);
    k_merge_init<<<dim3(NQ, BH), 128, 0, st>>>(mask, q_off, k_off, NQ, NK, Wd, m);
    PARK_TRY_LAUNCH("k_merge_init", st);
    ::park::prof_begin(st);
    k_merge_planes<<<BH, 128, 0, st>>>(k_off, NQ, NK, Wd, m);
    PARK_TRY_LAUNCH("k_merge_planes", st);
    return PARK_OK;
}

int launch_merge(uint8_t* mask, int32_t* kept_cnt, const int32_t* q_off, const int32_t* k_off, int BH, int N, int NQ,
                 int NK, int rounds, const MergeWs& m, int32_t* q_labels, int num_sms, cudaStream_t st) {
    const int Wd = (NK + 31) / 32;
    PARK_CHECK(launch_merge_setup(mask, q_off, k_off, BH, NQ, NK, m, st));
    const size_t sm = (size_t)kMergeGroups * kMergePlanes * Wd * 4;
    if (cudaFuncSetAttribute(k_merge_inter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess) {
        cudaGetLastError();
        return PARK_ERR_CUDA;
    }
    const dim3 gg((NQ + kMergeGroups - 1) / kMergeGroups, BH);
    for (int it = 0; it < rounds; ++it) {
        ::park::prof_begin(st);
        k_merge_inter<<<gg, 256, sm, st>>>(NQ, Wd, it == 0, m);
        PARK_TRY_LAUNCH("k_merge_inter", st);
        ::park::prof_begin(st);
        k_merge_pick<<<dim3((NQ + 7) / 8, BH), 256, 0, st>>>(NQ, m);
        PARK_TRY_LAUNCH("k_merge_pick", st);
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
