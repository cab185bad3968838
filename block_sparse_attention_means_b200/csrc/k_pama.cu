// PAMA block importance, top-p selection and the kept-block CSR.
//
// PAMA (PARK abstract; Figure 2 caption): every query i keeps its own Softmax
// over the non-empty key clusters, P_im = softmax_m(q_i . c_m / sqrt(D)), and
// I_rm is the mean of P_im over the members i of query cluster r.
//
// Fast path (bf16): k_pama_tc.cu computes the NQ x NK importance map on the
// tcgen05 tensor cores, streamed over the key centroids (per-query scores never
// reach memory: O(NQ*NK) extra memory, the streamed form of PARK Appendix
// Table 6), with a relative error bound rho_r for each row of I.
//
// top-p: per (query cluster, head) a bitonic sort (I descending, ties: lower m
// first) and a float64 prefix sum give the shortest prefix reaching p.  The
// decision is certified against rho_r; a row that is not certified is
// recomputed entirely in float64 (k_pama_f64), which also serves the float32
// input path for every row.
#include "kernels.h"

namespace park {

// ---------------------------------------------------------------- sort helpers
// Bitonic sort of n (power of two) (value, index) pairs: value descending,
// ties by index ascending.  All threads of the block take part (a multiple of
// 32).  Each stage (k, j) compares n / 2 pairs (i, i + j), pair q taking
// i = 2 (q - q mod j) + q mod j, so no thread only tests its index.  The 32
// pairs of a warp then touch one aligned block of 64 elements whenever j <= 32,
// so consecutive stages with j <= 32 need only a warp barrier; a block barrier
// separates every stage that crosses warps.
template <typename V>
__device__ void bitonic_desc(V* v, int32_t* idx, int n) {
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int q = threadIdx.x; q < (n >> 1); q += blockDim.x) {
                const int i = ((q & ~(j - 1)) << 1) | (q & (j - 1));
                const int ixj = i | j;
                const V a = v[i], b = v[ixj];
                const int ia = idx[i], ib = idx[ixj];
                const bool b_first = (b > a) || (b == a && ib < ia);
                const bool a_first = (a > b) || (a == b && ia < ib);
                const bool up = (i & k) == 0;
                if (up ? b_first : a_first) {
                    v[i] = b;
                    v[ixj] = a;
                    idx[i] = ib;
                    idx[ixj] = ia;
                }
            }
            const int jn = j > 1 ? j >> 1 : k;  // the next stage's j
            if (j > 32 || jn > 32 || (j == 1 && k == n))
                __syncthreads();
            else
                __syncwarp();
        }
    }
}

static int next_pow2(int x) {
    int p = 2;
    while (p < x) p <<= 1;
    return p;
}

// ---------------------------------------------------------------- top-p (certified)
__global__ __launch_bounds__(512) void k_topp(const float* __restrict__ importance, const float* __restrict__ rho,
                                              const int32_t* __restrict__ q_off, const int32_t* __restrict__ k_off,
                                              int NQ, int NK, int NKP, float p, int select,
                                              const float* __restrict__ sip_u, float* __restrict__ weight,
                                              uint8_t* __restrict__ mask, int32_t* __restrict__ kept_cnt,
                                              float* __restrict__ importance_bound, int32_t* __restrict__ flag_list,
                                              int32_t* __restrict__ flag_count) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    double* S = reinterpret_cast<double*>(smem_raw);       // [NKP] inclusive prefix sums
    float* sv = reinterpret_cast<float*>(S + NKP);         // [NKP]
    int32_t* si = reinterpret_cast<int32_t*>(sv + NKP);    // [NKP]
    uint8_t* keep = reinterpret_cast<uint8_t*>(si + NKP);  // [NKP]
    __shared__ double wsum[16];
    __shared__ int s_cut, s_live, s_t, s_bad, s_kept;

    const int r = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
    const size_t row = (size_t)bh * NQ + r;
    uint8_t* mrow = mask + row * NK;
    const int nr = q_off[(size_t)bh * (NQ + 1) + r + 1] - q_off[(size_t)bh * (NQ + 1) + r];
    if (nr == 0) {
        for (int m = t; m < NK; m += blockDim.x) {
            mrow[m] = 0;
            if (select == 2) weight[row * NK + m] = 0.f;
        }
        if (t == 0) {
            kept_cnt[row] = 0;
            if (importance_bound) importance_bound[row] = 0.f;
        }
        return;
    }
    const int32_t* ko = k_off + (size_t)bh * (NK + 1);
    const float* I = importance + row * NK;
    if (t == 0) {
        s_cut = -1;
        s_live = 0;
        s_t = 0x7fffffff;
        s_bad = 0;
        s_kept = 0;
    }
    __syncthreads();
    int live_local = 0;
    for (int m = t; m < NKP; m += blockDim.x) {
        bool lv = m < NK && ko[m + 1] > ko[m];
        sv[m] = lv ? I[m] : -1.0f;
        si[m] = m;
        keep[m] = 0;
        live_local += lv;
    }
    atomicAdd(&s_live, live_local);
    __syncthreads();
    bitonic_desc<float>(sv, si, NKP);
    const int L = s_live;
    // inclusive float64 prefix sums of the live sorted values
    const int seg = NKP / blockDim.x > 0 ? NKP / blockDim.x : 1;
    const int b0 = t * seg;
    double loc = 0.0;
    for (int e = b0; e < b0 + seg && e < NKP; ++e) loc += e < L ? (double)sv[e] : 0.0;
    // block exclusive scan of loc
    double incl = loc;
    const int lane = t & 31, w = t >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    if (t == 0) {
        double run = 0.0;
        for (int q = 0; q < (int)(blockDim.x >> 5); ++q) {
            double x = wsum[q];
            wsum[q] = run;
            run += x;
        }
    }
    __syncthreads();
    double run = wsum[w] + incl - loc;
    for (int e = b0; e < b0 + seg && e < NKP; ++e) {
        run += e < L ? (double)sv[e] : 0.0;
        S[e] = run;
    }
    __syncthreads();
    for (int e = t; e < L; e += blockDim.x)
        if (S[e] >= (double)p && (e == 0 || S[e - 1] < (double)p)) s_cut = e;
    __syncthreads();
    int cut = s_cut;
    bool ok;
    const double rh = (double)rho[row];
    if (select == 2) {
        // SIP: pi_e = 1 for the first tc sorted blocks, c sv[e] after them, with
        // sum pi = Bd; tc = first e with (Bd - e) sv[e] <= tail[e] (tail[e] = sum of
        // sv[e..L-1]).  Every decision is certified against the relative bound rh of
        // the float importances (a tail sum carries at most rh, c at most 2 rh), else
        // the whole row goes to float64.
        const int Bd = max(1, (int)ceil((double)p * (double)L));
        const double total = S[L - 1];
        auto tail = [&](int e) { return total - (e > 0 ? S[e - 1] : 0.0); };
        if (Bd < L)
            for (int e = t; e < L; e += blockDim.x)
                if ((double)(Bd - e) * (double)sv[e] <= tail(e)) atomicMin(&s_t, e);
        for (int m = t; m < NK; m += blockDim.x) weight[row * NK + m] = 0.f;
        __syncthreads();
        const int tc = Bd >= L ? L : s_t;
        double c = 0.0;
        if (tc < L) {
            c = (double)(Bd - tc) / tail(tc);
            if (t == 0) {
                bool b = !((double)(Bd - tc) * (double)sv[tc] * (1.0 + rh) < tail(tc) * (1.0 - rh));
                if (tc > 0) {
                    b |= !((double)(Bd - tc + 1) * (double)sv[tc - 1] * (1.0 - rh) > tail(tc - 1) * (1.0 + rh));
                    b |= !((double)sv[tc - 1] * (1.0 - rh) > (double)sv[tc] * (1.0 + 2.0 * rh));
                }
                if (b) s_bad = 1;
            }
        }
        int kept_local = 0;
        for (int e = t; e < L; e += blockDim.x) {
            const double pi = e < tc ? 1.0 : c * (double)sv[e];
            const int m = si[e];
            const double u = (double)sip_u[row * NK + m];
            if (e >= tc && fabs(u - pi) <= 4.0 * rh * pi + 1e-12) s_bad = 1;
            if (u < pi) {
                keep[m] = 1;
                weight[row * NK + m] = (float)(1.0 / pi);
                ++kept_local;
            }
        }
        atomicAdd(&s_kept, kept_local);
        __syncthreads();
        if (t == 0 && s_kept == 0) {  // nothing drawn: the most important block
            if (L > 1 && !((double)sv[0] * (1.0 - rh) > (double)sv[1] * (1.0 + 2.0 * rh))) s_bad = 1;
            const double pi0 = 0 < tc ? 1.0 : c * (double)sv[0];
            keep[si[0]] = 1;
            weight[row * NK + si[0]] = (float)(1.0 / pi0);
            s_kept = 1;
        }
        __syncthreads();
        ok = s_bad == 0;
        cut = s_kept - 1;
    } else if (select == 1) {  // the ceil(p L) most important; certified when the last kept is clear of the next
        const int kk = max(1, (int)ceil((double)p * (double)L));
        cut = min(kk, L) - 1;
        ok = cut + 1 >= L || (double)sv[cut] * (1.0 - rh) > (double)sv[cut + 1] * (1.0 + 2.0 * rh) + 1e-300;
    } else if (p >= 1.0f) {
        cut = L - 1;
        ok = true;
    } else if (cut < 0) {
        ok = false;  // float sums fell short of p: let float64 decide
    } else {
        // The exact importances of a row sum to 1 (every query's Softmax does), so the
        // error of a running sum is minus the error of what lies after it: with
        // T = sum of every computed value and each value within rh of the exact one
        // (relative), the exact running sum through sorted position e lies within
        // rh / (1 - rh) (T - S[e]) of S[e] - (T - 1).  After the cut only about 1 - p
        // of the mass is left, so this is about (1 - p) / p times the plain bound.
        // The order of the last kept and the first dropped value is certain when
        // the exact values, each within re of the computed one, cannot swap.
        const double vc = (double)sv[cut];
        const double eps = 1e-12;
        const double re = rh + 0x1p-23;  // + the float rounding of the stored values
        const double T = S[L - 1], E = T - 1.0, rp = re / (1.0 - re);
        const double Sc = S[cut], Sb = cut > 0 ? S[cut - 1] : 0.0;
        bool ord = cut + 1 >= L || vc * (1.0 - re) > (double)sv[cut + 1] * (1.0 + re) + 1e-300;
        bool hi = Sc - E - rp * (T - Sc) - eps >= (double)p;  // the exact sum through the cut reaches p
        bool lo = Sb - E + rp * (T - Sb) + eps < (double)p;   // and the one before it does not
        ok = rh < 0.5 && ord && hi && lo;
    }
    if (!ok) {
        if (t == 0) {
            int pos = atomicAdd(flag_count, 1);
            flag_list[pos] = (int32_t)row;
        }
        return;
    }
    if (select != 2)
        for (int e = t; e <= cut; e += blockDim.x) keep[si[e]] = 1;
    __syncthreads();
    for (int m = t; m < NK; m += blockDim.x) mrow[m] = keep[m];
    if (t == 0) {
        kept_cnt[row] = cut + 1;
        if (importance_bound) importance_bound[row] = rho[row];
    }
}

int launch_topp(const float* importance, const float* rho, int BH, int NQ, int NK, const int32_t* q_off,
                const int32_t* k_off, float p, int select, const float* sip_u, float* weight, uint8_t* mask,
                int32_t* kept_cnt, float* importance_bound, int32_t* flag_list, int32_t* flag_count,
                cudaStream_t st) {
    int NKP = next_pow2(NK);
    if (NKP < 512) NKP = 512;
    size_t sm = (size_t)NKP * (8 + 4 + 4 + 1) + 16;
    cudaFuncSetAttribute(k_topp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    ::park::prof_begin(st);
    k_topp<<<dim3(NQ, BH), 512, sm, st>>>(importance, rho, q_off, k_off, NQ, NK, NKP, p, select, sip_u, weight,
                                          mask, kept_cnt,
                                          importance_bound, flag_list, flag_count);
    PARK_TRY_LAUNCH("k_topp", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- float64 PAMA + top-p
// One CTA (256 threads) per listed (head, query cluster), or per cluster of
// every head when all_clusters is set; CTAs take clusters from an atomic work
// counter.  The cluster's rows are staged RT at a time in shared memory as
// float64, transposed (Qs[k][row]); the key centroids stream through in
// chunks of 64 (Cs[k][col]), the next chunk prefetched through registers while
// the current one is used.  Thread (ty, tx) of a 16 x 16 grid owns the RPT x 4
// logit block rows ty*RPT + i, columns 4*tx + u of the RT x 64 tile (RT = 16
// RPT), read with 16-byte shared loads.
//   pass 1: logits z (scaled; -inf for empty key clusters) into the CTA's
//           float64 scratch, and the row max;
//   pass 2: e = exp(z - max) over the scratch, row sums;
//   pass 3: P = e / sum, summed over the rows into per-row-group column
//           partials that are added in a fixed order.
// Then I = column sums / |Q_r| is sorted (descending, ties by m) and a
// sequential float64 running sum finds the cut, as the definition reads.
constexpr int F64_CH = 64;  // centroids per chunk

template <typename T, int RPT>
__global__ __launch_bounds__(256, 1) void k_pama_f64(const T* __restrict__ Q, const int32_t* __restrict__ q_perm,
                                                     const int32_t* __restrict__ q_off, const T* __restrict__ CK,
                                                     const int32_t* __restrict__ k_off, int N, int D, int NQ, int NK,
                                                     int NKP, double scale, float p, int select, int size_prior,
                                                     const float* __restrict__ sip_u, float* __restrict__ weight,
                                                     const int32_t* __restrict__ list,
                                                     const int32_t* __restrict__ count_ptr, int all_clusters,
                                                     int BHNQ, int32_t* __restrict__ work_ctr,
                                                     double* __restrict__ zscratch, float* __restrict__ importance,
                                                     float* __restrict__ importance_bound,
                                                     uint8_t* __restrict__ mask, int32_t* __restrict__ kept_cnt,
                                                     int64_t* __restrict__ counters) {
    constexpr int RT = 16 * RPT, DM = 128, ZB = RPT * 4;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    double* Qs = reinterpret_cast<double*>(smem_raw);          // [DM][RT]
    double* Cs = Qs + DM * RT;                                 // [DM][F64_CH]
    double* Isum = Cs + DM * F64_CH;                           // [NKP]
    double* part = Isum + NKP;                                 // [16][F64_CH]
    double* lsz = part + 16 * F64_CH;                          // [NKP] additive logit term per column
    int32_t* si = reinterpret_cast<int32_t*>(lsz + NKP);       // [NKP]
    uint8_t* live = reinterpret_cast<uint8_t*>(si + NKP);      // [NKP]
    __shared__ int s_cut, s_e, s_tc, s_kept;
    __shared__ double s_c;
    const double NEG_INF = __longlong_as_double(0xfff0000000000000ll);
    const int t = threadIdx.x, ty = t >> 4, tx = t & 15;
    const int count = all_clusters ? BHNQ : *count_ptr;
    if (blockIdx.x == 0 && t == 0 && !all_clusters && counters)
        atomicAdd((unsigned long long*)(counters + PARK_CNT_PAMA_RECHECK), (unsigned long long)count);
    const int nch = (NK + F64_CH - 1) / F64_CH;
    double* zs = zscratch + (size_t)blockIdx.x * nch * 256 * ZB;  // this CTA's scratch
    // chunk staging: thread t holds centroid (t >> 2) of the chunk, dims (t & 3) + 4 v
    constexpr int CPT = F64_CH * DM / 256;  // elements per thread (32)
    for (;;) {
        __syncthreads();  // previous entry's shared memory fully consumed
        if (t == 0) s_e = atomicAdd(work_ctr, 1);
        __syncthreads();
        const int e = s_e;
        if (e >= count) break;
        const int row = all_clusters ? e : list[e];
        const int bh = row / NQ, r = row - bh * NQ;
        const int qs = q_off[(size_t)bh * (NQ + 1) + r], nr = q_off[(size_t)bh * (NQ + 1) + r + 1] - qs;
        const int32_t* ko = k_off + (size_t)bh * (NK + 1);
        uint8_t* mrow = mask + (size_t)row * NK;
        float* Irow = importance + (size_t)row * NK;
        if (nr == 0) {
            for (int m = t; m < NK; m += blockDim.x) {
                mrow[m] = 0;
                Irow[m] = 0.f;
                if (select == 2) weight[(size_t)row * NK + m] = 0.f;
            }
            if (t == 0) {
                kept_cnt[row] = 0;
                if (importance_bound) importance_bound[row] = 0.f;
            }
            continue;
        }
        for (int m = t; m < NKP; m += blockDim.x) {
            Isum[m] = 0.0;
            const int nm = m < NK ? ko[m + 1] - ko[m] : 0;
            live[m] = nm > 0 ? 1 : 0;
            lsz[m] = (size_prior && nm > 0) ? log((double)nm) : 0.0;  // the size prior log |B_m|
        }
        const T* Ch = CK + (size_t)bh * NK * D;
        const T* Qh = Q + (size_t)bh * N * D;
        const int32_t* pm = q_perm + (size_t)bh * N + qs;
        float cpre[CPT];  // inputs are exact in float32 (bf16 or float32)
        auto fetch_chunk = [&](int c) {  // global -> registers
            const int m = c * F64_CH + (t >> 2);
#pragma unroll
            for (int v = 0; v < CPT; ++v) {
                const int k = (t & 3) + 4 * v;
                cpre[v] = (m < NK && k < D) ? Elem<T>::to_float(Ch + (size_t)m * D, k) : 0.f;
            }
        };
        auto store_chunk = [&]() {  // registers -> Cs[k][col]
            const int col = t >> 2;
#pragma unroll
            for (int v = 0; v < CPT; ++v) Cs[((t & 3) + 4 * v) * F64_CH + col] = (double)cpre[v];
        };
        for (int t0 = 0; t0 < nr; t0 += RT) {
            __syncthreads();  // Qs free
            for (int idx = t; idx < RT * DM; idx += blockDim.x) {
                const int k = idx / RT, rr = idx - k * RT;
                Qs[k * RT + rr] = (t0 + rr < nr && k < D) ? Elem<T>::to_double(Qh + (size_t)pm[t0 + rr] * D, k) : 0.0;
            }
            // pass 1: logits into the scratch, row max
            double mx[RPT];
#pragma unroll
            for (int i = 0; i < RPT; ++i) mx[i] = NEG_INF;
            fetch_chunk(0);
            for (int c = 0; c < nch; ++c) {
                __syncthreads();  // Cs free (and Qs staged)
                store_chunk();
                __syncthreads();
                if (c + 1 < nch) fetch_chunk(c + 1);  // in flight during the GEMM
                double z[RPT][4];
#pragma unroll
                for (int i = 0; i < RPT; ++i)
#pragma unroll
                    for (int u = 0; u < 4; ++u) z[i][u] = 0.0;
#pragma unroll 2
                for (int k = 0; k < DM; ++k) {
                    double a[RPT], b[4];
#pragma unroll
                    for (int i = 0; i < RPT; i += 2) {
                        const double2 q2 = *reinterpret_cast<const double2*>(Qs + k * RT + ty * RPT + i);
                        a[i] = q2.x;
                        a[i + 1] = q2.y;
                    }
                    const double2 c0 = *reinterpret_cast<const double2*>(Cs + k * F64_CH + 4 * tx);
                    const double2 c1 = *reinterpret_cast<const double2*>(Cs + k * F64_CH + 4 * tx + 2);
                    b[0] = c0.x;
                    b[1] = c0.y;
                    b[2] = c1.x;
                    b[3] = c1.y;
#pragma unroll
                    for (int i = 0; i < RPT; ++i)
#pragma unroll
                        for (int u = 0; u < 4; ++u) z[i][u] = __fma_rn(a[i], b[u], z[i][u]);
                }
                double2* zb = reinterpret_cast<double2*>(zs + ((size_t)c * 256 + t) * ZB);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int col = c * F64_CH + 4 * tx + u;
                    const bool lv = col < NK && live[col];
#pragma unroll
                    for (int i = 0; i < RPT; ++i) {
                        z[i][u] = lv ? scale * z[i][u] + lsz[col] : NEG_INF;
                        mx[i] = fmax(mx[i], z[i][u]);
                    }
                }
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    zb[2 * i] = make_double2(z[i][0], z[i][1]);
                    zb[2 * i + 1] = make_double2(z[i][2], z[i][3]);
                }
            }
#pragma unroll
            for (int i = 0; i < RPT; ++i)
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) mx[i] = fmax(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], o, 16));
            // pass 2: e = exp(z - max) over this thread's own scratch blocks, row sums
            double sm[RPT];
#pragma unroll
            for (int i = 0; i < RPT; ++i) sm[i] = 0.0;
            for (int c = 0; c < nch; ++c) {
                double2* zb = reinterpret_cast<double2*>(zs + ((size_t)c * 256 + t) * ZB);
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    double2 v0 = zb[2 * i], v1 = zb[2 * i + 1];
                    v0.x = exp(v0.x - mx[i]);
                    v0.y = exp(v0.y - mx[i]);
                    v1.x = exp(v1.x - mx[i]);
                    v1.y = exp(v1.y - mx[i]);
                    sm[i] += (v0.x + v0.y) + (v1.x + v1.y);
                    zb[2 * i] = v0;
                    zb[2 * i + 1] = v1;
                }
            }
            double inv[RPT];
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) sm[i] += __shfl_xor_sync(0xffffffffu, sm[i], o, 16);
                inv[i] = (t0 + ty * RPT + i < nr) ? 1.0 / sm[i] : 0.0;
            }
            // pass 3: normalised probabilities summed over the tile's rows
            for (int c = 0; c < nch; ++c) {
                const double2* zb = reinterpret_cast<const double2*>(zs + ((size_t)c * 256 + t) * ZB);
                double cs[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    const double2 v0 = zb[2 * i], v1 = zb[2 * i + 1];
                    cs[0] += v0.x * inv[i];
                    cs[1] += v0.y * inv[i];
                    cs[2] += v1.x * inv[i];
                    cs[3] += v1.y * inv[i];
                }
                __syncthreads();  // part free
#pragma unroll
                for (int u = 0; u < 4; ++u) part[ty * F64_CH + 4 * tx + u] = cs[u];
                __syncthreads();
                if (t < F64_CH) {
                    double s = 0.0;
                    for (int q = 0; q < 16; ++q) s += part[q * F64_CH + t];
                    const int col = c * F64_CH + t;
                    if (col < NK) Isum[col] += s;
                }
            }
        }
        __syncthreads();
        for (int m = t; m < NKP; m += blockDim.x) {
            const bool lv = live[m] != 0;
            const double iv = lv ? Isum[m] / (double)nr : -1.0;
            if (m < NK) Irow[m] = lv ? (float)iv : 0.f;
            Isum[m] = iv;
            si[m] = m;
        }
        __syncthreads();
        bitonic_desc<double>(Isum, si, NKP);
        if (select == 2) {
            // SIP in float64, as the definition reads: tail sums from the smallest up,
            // the first sorted position whose (Bd - t) v_t fits under its tail, then
            // one draw per block against the caller's uniform
            double* tail = lsz;  // free after the GEMM passes
            if (t == 0) {
                int L = 0;
                while (L < NKP && Isum[L] >= 0.0) ++L;
                const int Bd = max(1, (int)ceil((double)p * (double)L));
                int tc = L;
                double c = 0.0;
                if (Bd < L) {
                    tail[L - 1] = Isum[L - 1];
                    for (int e = L - 2; e >= 0; --e) tail[e] = tail[e + 1] + Isum[e];
                    tc = 0;
                    while ((double)(Bd - tc) * Isum[tc] > tail[tc]) ++tc;
                    c = (double)(Bd - tc) / tail[tc];
                }
                s_cut = L;
                s_tc = tc;
                s_c = c;
                s_kept = 0;
                if (importance_bound) importance_bound[row] = 0.f;
            }
            for (int m = t; m < NK; m += blockDim.x) {
                mrow[m] = 0;
                weight[(size_t)row * NK + m] = 0.f;
            }
            __syncthreads();
            const int L = s_cut, tc = s_tc;
            const double c = s_c;
            int kept_local = 0;
            for (int e = t; e < L; e += blockDim.x) {
                const double pi = e < tc ? 1.0 : c * Isum[e];
                const int m = si[e];
                if ((double)sip_u[(size_t)row * NK + m] < pi) {
                    mrow[m] = 1;
                    weight[(size_t)row * NK + m] = (float)(1.0 / pi);
                    ++kept_local;
                }
            }
            atomicAdd(&s_kept, kept_local);
            __syncthreads();
            if (t == 0) {
                if (s_kept == 0) {  // nothing drawn: the most important block
                    const double pi0 = 0 < tc ? 1.0 : c * Isum[0];
                    mrow[si[0]] = 1;
                    weight[(size_t)row * NK + si[0]] = (float)(1.0 / pi0);
                    s_kept = 1;
                }
                kept_cnt[row] = s_kept;
            }
            continue;
        }
        if (t == 0) {
            double run = 0.0;
            int cut = -1;
            if (select == 1) {  // the ceil(p L) most important of the L non-empty key clusters
                int L = 0;
                while (L < NKP && Isum[L] >= 0.0) ++L;
                cut = L > 0 ? min(max(1, (int)ceil((double)p * (double)L)), L) - 1 : -1;
            } else {
                for (int q = 0; q < NKP && Isum[q] >= 0.0; ++q) {
                    cut = q;
                    run += Isum[q];
                    if (p < 1.0f && run >= (double)p) break;
                }
            }
            s_cut = cut;
            kept_cnt[row] = cut + 1;
            if (importance_bound) importance_bound[row] = 0.f;
        }
        __syncthreads();
        const int cut = s_cut;
        for (int m = t; m < NK; m += blockDim.x) mrow[m] = 0;
        __syncthreads();
        for (int q = t; q <= cut; q += blockDim.x) mrow[si[q]] = 1;
    }
}

size_t pama_f64_scratch_bytes(int NK) {
    return (size_t)kPamaF64Slots * ((NK + F64_CH - 1) / F64_CH) * 256 * 32 * sizeof(double);
}

template <typename T, int RPT>
static void pama_f64_launch(const void* Q, const int32_t* q_perm, const int32_t* q_off, const void* CK,
                            const int32_t* k_off, int N, int D, int NQ, int NK, int NKP, double scale, float p,
                            int select, int size_prior, const float* sip_u, float* weight, const int32_t* list,
                            const int32_t* count, int all_clusters, int BHNQ, int32_t* work_ctr,
                            double* zscratch, float* importance, float* importance_bound, uint8_t* mask,
                            int32_t* kept_cnt, int64_t* counters, size_t sm, int blocks, cudaStream_t st) {
    cudaFuncSetAttribute(k_pama_f64<T, RPT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_pama_f64<T, RPT><<<blocks, 256, sm, st>>>((const T*)Q, q_perm, q_off, (const T*)CK, k_off, N, D, NQ, NK, NKP,
                                                scale, p, select, size_prior, sip_u, weight, list, count,
                                                all_clusters, BHNQ,
                                                work_ctr, zscratch,
                                                importance, importance_bound, mask, kept_cnt, counters);
}

int launch_pama_f64(const void* Q, int dtype, int BH, int N, int D, int NQ, int NK, const int32_t* q_perm,
                    const int32_t* q_off, const void* CK, const int32_t* k_off, float p, int select, int size_prior,
                    const float* sip_u, float* weight, const int32_t* list,
                    const int32_t* count, int all_clusters, int num_sms, int32_t* work_ctr, double* zscratch,
                    float* importance, float* importance_bound, uint8_t* mask, int32_t* kept_cnt, int64_t* counters,
                    cudaStream_t st, int one_row) {
    if (NK > 4096 || D > 128) return PARK_ERR_UNSUPPORTED;
    const int NKP = next_pow2(NK);
    auto smem = [&](int RT) {
        return (size_t)128 * RT * 8 + (size_t)128 * F64_CH * 8 + (size_t)NKP * 8 + 16 * F64_CH * 8 + (size_t)NKP * 8 +
               (size_t)NKP * 4 + NKP;
    };
    // 128-row tiles when the sort buffers leave room; 32-row tiles when every
    // cluster is a single row (the query centroids of "w/o PAMA")
    const bool big = smem(128) <= 227 * 1024 && !one_row;
    const size_t sm = smem(one_row ? 32 : big ? 128 : 64);
    const int blocks = num_sms < kPamaF64Slots ? num_sms : kPamaF64Slots;
    const double scale = 1.0 / sqrt((double)D);
    ::park::prof_begin(st);
    if (one_row) {
        if (dtype == PARK_BF16)
            pama_f64_launch<bf16_t, 2>(Q, q_perm, q_off, CK, k_off, N, D, NQ, NK, NKP, scale, p, select, size_prior,
                                       sip_u, weight, list, count, all_clusters, BH * NQ, work_ctr, zscratch,
                                       importance, importance_bound, mask, kept_cnt, counters, sm, blocks, st);
        else
            pama_f64_launch<float, 2>(Q, q_perm, q_off, CK, k_off, N, D, NQ, NK, NKP, scale, p, select, size_prior,
                                      sip_u, weight, list, count, all_clusters, BH * NQ, work_ctr, zscratch,
                                      importance, importance_bound, mask, kept_cnt, counters, sm, blocks, st);
    } else if (dtype == PARK_BF16) {
        if (big)
            pama_f64_launch<bf16_t, 8>(Q, q_perm, q_off, CK, k_off, N, D, NQ, NK, NKP, scale, p, select, size_prior, sip_u, weight, list, count,
                                       all_clusters, BH * NQ, work_ctr, zscratch, importance, importance_bound, mask,
                                       kept_cnt, counters, sm, blocks, st);
        else
            pama_f64_launch<bf16_t, 4>(Q, q_perm, q_off, CK, k_off, N, D, NQ, NK, NKP, scale, p, select, size_prior, sip_u, weight, list, count,
                                       all_clusters, BH * NQ, work_ctr, zscratch, importance, importance_bound, mask,
                                       kept_cnt, counters, sm, blocks, st);
    } else {
        if (big)
            pama_f64_launch<float, 8>(Q, q_perm, q_off, CK, k_off, N, D, NQ, NK, NKP, scale, p, select, size_prior, sip_u, weight, list, count,
                                      all_clusters, BH * NQ, work_ctr, zscratch, importance, importance_bound, mask,
                                      kept_cnt, counters, sm, blocks, st);
        else
            pama_f64_launch<float, 4>(Q, q_perm, q_off, CK, k_off, N, D, NQ, NK, NKP, scale, p, select, size_prior, sip_u, weight, list, count,
                                      all_clusters, BH * NQ, work_ctr, zscratch, importance, importance_bound, mask,
                                      kept_cnt, counters, sm, blocks, st);
    }
    PARK_TRY_LAUNCH("k_pama_f64", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- "w/o PAMA" rows
// Rows for the float64 PAMA kernel when the query centroid stands for its
// cluster: cluster r has one row (centroid r) if it is non-empty, none
// otherwise.  off[r] = number of non-empty clusters before r, perm[off[r]] = r.
__global__ __launch_bounds__(1024) void k_centroid_rows(const int32_t* __restrict__ q_off, int NQ,
                                                        int32_t* __restrict__ perm, int32_t* __restrict__ off) {
    __shared__ int32_t wsum[32];
    const int bh = blockIdx.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int32_t* qo = q_off + (size_t)bh * (NQ + 1);
    int32_t* po = off + (size_t)bh * (NQ + 1);
    int32_t* pp = perm + (size_t)bh * NQ;
    const int seg = (NQ + 1023) / 1024, b0 = t * seg, b1 = min(NQ, b0 + seg);
    int loc = 0;
    for (int r = b0; r < b1; ++r) loc += qo[r + 1] > qo[r];
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
    for (int r = b0; r < b1; ++r) {
        po[r] = run;
        if (qo[r + 1] > qo[r]) pp[run++] = r;
    }
    if (b0 < NQ && b1 == NQ) po[NQ] = run;
    if (NQ == 0 && t == 0) po[0] = 0;
}

int launch_centroid_rows(const int32_t* q_off, int BH, int NQ, int32_t* perm, int32_t* off, cudaStream_t st) {
    ::park::prof_begin(st);
    k_centroid_rows<<<BH, 1024, 0, st>>>(q_off, NQ, perm, off);
    PARK_TRY_LAUNCH("k_centroid_rows", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- kept-block CSR
__global__ __launch_bounds__(1024) void k_kept_scan(const int32_t* __restrict__ cnt, int NQ,
                                                    int32_t* __restrict__ ptr, int64_t* __restrict__ counters) {
    __shared__ int wsum[32];
    const int bh = blockIdx.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int seg = (NQ + 1023) / 1024, b0 = t * seg;
    const int32_t* c = cnt + (size_t)bh * NQ;
    int loc = 0;
    for (int e = b0; e < b0 + seg && e < NQ; ++e) loc += c[e];
    int incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    if (w == 0) {
        int x = wsum[lane], xi = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, xi, o);
            if (lane >= o) xi += y;
        }
        wsum[lane] = xi - x;
    }
    __syncthreads();
    int run = wsum[w] + incl - loc;
    int32_t* pr = ptr + (size_t)bh * (NQ + 1);
    for (int e = b0; e < b0 + seg && e < NQ; ++e) {
        pr[e] = run;
        run += c[e];
    }
    if (b0 < NQ && b0 + seg >= NQ) {
        pr[NQ] = run;
        if (counters) atomicAdd((unsigned long long*)(counters + PARK_CNT_KEPT_BLOCKS), (unsigned long long)run);
    }
}

__global__ __launch_bounds__(256) void k_kept_compact(const uint8_t* __restrict__ mask, const int32_t* __restrict__ ptr,
                                                      int NQ, int NK, int32_t* __restrict__ idx) {
    __shared__ int wcnt[8];
    const int r = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const uint8_t* mrow = mask + ((size_t)bh * NQ + r) * NK;
    int32_t* out = idx + (size_t)bh * NQ * NK + ptr[(size_t)bh * (NQ + 1) + r];
    int base = 0;
    for (int m0 = 0; m0 < NK; m0 += 256) {
        int m = m0 + t;
        bool f = m < NK && mrow[m];
        unsigned bal = __ballot_sync(0xffffffffu, f);
        if (lane == 0) wcnt[w] = __popc(bal);
        __syncthreads();
        int off = base;
        for (int q = 0; q < w; ++q) off += wcnt[q];
        if (f) out[off + __popc(bal & ((1u << lane) - 1u))] = m;
        int tot = 0;
        for (int q = 0; q < 8; ++q) tot += wcnt[q];
        base += tot;
        __syncthreads();
    }
}

int launch_kept_csr(const uint8_t* mask, const int32_t* kept_cnt, int BH, int NQ, int NK, int32_t* kept_ptr,
                    int32_t* kept_idx, int64_t* counters, cudaStream_t st) {
    ::park::prof_begin(st);
    k_kept_scan<<<BH, 1024, 0, st>>>(kept_cnt, NQ, kept_ptr, counters);
    PARK_TRY_LAUNCH("k_kept_scan", st);
    ::park::prof_begin(st);
    k_kept_compact<<<dim3(NQ, BH), 256, 0, st>>>(mask, kept_ptr, NQ, NK, kept_idx);
    PARK_TRY_LAUNCH("k_kept_compact", st);
    return PARK_OK;
}

}  // namespace park
