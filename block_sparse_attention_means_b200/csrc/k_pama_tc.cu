// PAMA block importance on the 5th-generation tensor cores (tcgen05 + TMEM +
// TMA), bf16 inputs, D = 128.
//
// PAMA (PARK abstract; Figure 2 caption): every query i keeps its own Softmax
// over the non-empty key clusters, P_im = softmax_m(q_i . c_m / sqrt(D)), and
// I_rm is the mean of P_im over the members i of query cluster r.
//
// Work item = one query cluster (persistent CTAs, round-robin).  Its rows,
// gathered into cluster order beforehand, are taken in 128-row tiles (TMA); the
// key centroids stream in chunks of 128 (TMA, 2-stage ring), twice per tile:
// pass 1 gives every row its maximum logit and Softmax denominator, pass 2 the
// normalised probabilities, summed over the tile's rows into per-cluster column
// sums.  S = Q C^T of a chunk goes to one of four TMEM buffers (128 x 128 fp32).
//
// Warps: 0 loads, 1 owns TMEM and issues the MMAs (one thread), 2-9 are two
// epilogue groups of four warps (one thread per row, all 128 columns of a
// chunk) that take the chunk MMAs alternately, so one group's exponentials
// overlap the other's TMEM loads.  In pass 1 each group keeps its own running
// (max, sum) per row; the two meet through shared memory before pass 2.  The
// column sums of a chunk over a warp's 32 rows come from a transposing
// shuffle reduction (lane j ends with column j).
//
// Error bound rho_r (relative, for the row I_r.) as for the warp-level kernel:
// the logit error of the fp32 tensor-core accumulation (the kappa model), the
// exp2 approximations, the float32 row-sum partials (8 x 8 terms per 64
// columns, then float64) and the float32 column sums.
//
// Every wait is time-bounded (PARK_ERR_TIMEOUT on expiry); epilogue warps never
// leave their loops early (after a failed wait they only skip the waits).
#include "kernels.h"
#include "sm100.cuh"

namespace park {

using namespace sm100;

namespace {
constexpr int PT_ROWS = 128, PT_CH = 128, PT_BLK = 16384, PT_NB = 4;
constexpr uint32_t PT_TMEM_COLS = 512;  // PT_NB accumulators of 128 columns

struct PtSmem {
    uint64_t q_full, q_empty, c_full[2], c_empty[2], acc_full[PT_NB], acc_empty[PT_NB], final_bar;
    uint32_t tmem_base;
    int abort;
    float xm[2][PT_ROWS];   // [group][row] pass-1 maximum (log2 units)
    double xl[2][PT_ROWS];  // [group][row] pass-1 sum relative to it
    float sdmax[8];
};

__device__ __forceinline__ float fast_exp2(float x) { return exp2f(x); }
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Sum of v[0..31] over the 32 lanes of the warp: lane j returns the total of
// element j (31 shuffles, recursive halving).
__device__ __forceinline__ float transpose_sum32(float (&v)[32], int lane) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int k = 0; k < o; ++k) {
            const float send = upper ? v[k] : v[k + o];
            const float keep = upper ? v[k + o] : v[k];
            v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}
}  // namespace

__global__ void __launch_bounds__(320, 1)
    k_pama_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC,
              const int32_t* __restrict__ q_perm, const int32_t* __restrict__ q_off,
              const int32_t* __restrict__ k_off, const float* __restrict__ qnorm, const float* __restrict__ ckmax,
              int N, int NQ, int NK, int BH, float sl2e, float delta_scale, int size_prior,
              float* __restrict__ importance, float* __restrict__ rho, int32_t* __restrict__ status,
              uint64_t wait_ns) {
    extern __shared__ __align__(1024) uint8_t dsmem_raw[];
    __shared__ PtSmem sh;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Qs = base;                // 2 column blocks of the row tile
    uint8_t* Cs = base + 2 * PT_BLK;   // 2 stages x 2 column blocks
    const int nch = (NK + PT_CH - 1) / PT_CH;
    float* live = reinterpret_cast<float*>(Cs + 4 * PT_BLK);  // [nch*128] additive log2 term, -inf if empty
    float* colsum = live + nch * PT_CH;                        // [4][nch*128] per TMEM lane quadrant
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort = &sh.abort;
    if (threadIdx.x == 0) {
        mbar_init(&sh.q_full, 1);
        mbar_init(&sh.q_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.c_full[s], 1);
            mbar_init(&sh.c_empty[s], 1);
        }
        for (int b = 0; b < PT_NB; ++b) {
            mbar_init(&sh.acc_full[b], 1);
            mbar_init(&sh.acc_empty[b], 128);
        }
        mbar_init(&sh.final_bar, 1);
        sh.abort = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(&sh.tmem_base, PT_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int n_items = BH * NQ;
    const uint32_t idS = idesc_bf16(128, 128, 0, 0);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int G = 0, I = 0, c_last[2] = {-1, -1}, q_last = -1;
            bool ok = true;
            for (int it = blockIdx.x; it < n_items && ok && !*abort; it += gridDim.x) {
                const int bh = it / NQ, r = it - bh * NQ;
                const int qs = q_off[(size_t)bh * (NQ + 1) + r], nr = q_off[(size_t)bh * (NQ + 1) + r + 1] - qs;
                for (int t0 = 0; t0 < nr && ok; t0 += PT_ROWS) {
                    if (I > 0 && !mbar_wait(&sh.q_empty, (I - 1) & 1, abort, wait_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.q_full, 2 * PT_BLK);
                    tma_load_2d(Qs, &tmQ, &sh.q_full, 0, bh * N + qs + t0);
                    tma_load_2d(Qs + PT_BLK, &tmQ, &sh.q_full, 64, bh * N + qs + t0);
                    q_last = I & 1;
                    for (int c2 = 0; c2 < 2 * nch; ++c2) {  // both passes
                        const int c = c2 < nch ? c2 : c2 - nch;
                        const int s = G & 1, round = G >> 1;
                        if (round > 0 && !mbar_wait(&sh.c_empty[s], (round - 1) & 1, abort, wait_ns)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&sh.c_full[s], 2 * PT_BLK);
                        tma_load_2d(Cs + 2 * s * PT_BLK, &tmC, &sh.c_full[s], 0, bh * NK + c * PT_CH);
                        tma_load_2d(Cs + (2 * s + 1) * PT_BLK, &tmC, &sh.c_full[s], 64, bh * NK + c * PT_CH);
                        c_last[s] = round & 1;
                        ++G;
                    }
                    ++I;
                }
            }
            int dummy = 0;
            for (int s = 0; s < 2; ++s)
                if (c_last[s] >= 0) mbar_wait(&sh.c_full[s], c_last[s], &dummy, 100000000ull);
            if (q_last >= 0) mbar_wait(&sh.q_full, q_last, &dummy, 100000000ull);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int G = 0, I = 0;
            bool ok = true;
            const uint32_t qa = smem_u32(Qs);
            for (int it = blockIdx.x; it < n_items && ok && !*abort; it += gridDim.x) {
                const int bh = it / NQ, r = it - bh * NQ;
                const int nr = q_off[(size_t)bh * (NQ + 1) + r + 1] - q_off[(size_t)bh * (NQ + 1) + r];
                for (int t0 = 0; t0 < nr && ok; t0 += PT_ROWS) {
                    if (!mbar_wait(&sh.q_full, I & 1, abort, wait_ns)) {
                        ok = false;
                        break;
                    }
                    for (int c2 = 0; c2 < 2 * nch; ++c2) {
                        const int s = G & 1, b = G % PT_NB;
                        if (!mbar_wait(&sh.c_full[s], (G >> 1) & 1, abort, wait_ns) ||
                            (G >= PT_NB && !mbar_wait(&sh.acc_empty[b], (G / PT_NB - 1) & 1, abort, wait_ns))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t ca = smem_u32(Cs + 2 * s * PT_BLK);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t off = (uint32_t)((kk >> 2) * PT_BLK + (kk & 3) * 32);
                            umma_bf16(tmem + (uint32_t)(b * 128), sdesc_sw128(qa + off, 16, 1024),
                                      sdesc_sw128(ca + off, 16, 1024), idS, kk > 0);
                        }
                        umma_commit(&sh.acc_full[b]);
                        umma_commit(&sh.c_empty[s]);
                        ++G;
                    }
                    if (!ok) break;
                    umma_commit(&sh.q_empty);
                    ++I;
                }
            }
            umma_commit(&sh.final_bar);
            int dummy = 0;
            mbar_wait(&sh.final_bar, 0, &dummy, 100000000ull);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int grp = (warp - 2) >> 2, quad = warp & 3;
        const int row = 32 * quad + lane;
        const uint32_t trow = tmem + ((uint32_t)(32 * quad) << 16);
        const int et = threadIdx.x - 64;  // 0..255
        const float NEG = __int_as_float(0xff800000);
        const float2 sl2e2 = make_float2(sl2e, sl2e);
        bool failed = false;
        int G = 0;
        auto wait_acc = [&](int b, int g) {
            if (!failed) failed = !__all_sync(0xffffffffu, mbar_wait(&sh.acc_full[b], (g / PT_NB) & 1, abort, wait_ns));
            tc_fence_after();
        };
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const int bh = it / NQ, r = it - bh * NQ;
            const int qs = q_off[(size_t)bh * (NQ + 1) + r], nr = q_off[(size_t)bh * (NQ + 1) + r + 1] - qs;
            float* Irow = importance + (size_t)it * NK;
            if (nr == 0) {
                for (int m = et; m < NK; m += 256) Irow[m] = 0.f;
                if (et == 0) rho[it] = 0.f;
                continue;
            }
            // the head's additive column terms; zeroed column sums
            const int32_t* ko = k_off + (size_t)bh * (NK + 1);
            named_bar_sync(1, 256);
            for (int m = et; m < nch * PT_CH; m += 256) {
                const int sz = m < NK ? ko[m + 1] - ko[m] : 0;
                live[m] = sz > 0 ? (size_prior ? (float)log2((double)sz) : 0.f) : NEG;
#pragma unroll
                for (int q = 0; q < 4; ++q) colsum[q * nch * PT_CH + m] = 0.f;
            }
            named_bar_sync(1, 256);
            float dmax = 0.f;
            for (int t0 = 0; t0 < nr; t0 += PT_ROWS) {
                const bool valid = t0 + row < nr;
                if (valid && grp == 0) dmax = fmaxf(dmax, qnorm[(size_t)bh * N + q_perm[(size_t)bh * N + qs + t0 + row]]);
                // pass 1: this group's running maximum and sum of its chunks
                float m = NEG;
                double l = 0.0;
                for (int c = 0; c < nch; ++c, ++G) {
                    if ((G & 1) != grp) continue;
                    const int b = G % PT_NB;
                    wait_acc(b, G);
                    float x[2][32];
                    float cm = NEG;
                    float part[8];  // 8 partial sums of 8 terms per 64 columns: error <= (7 + 3) 2^-24
#pragma unroll
                    for (int h = 0; h < 2; ++h) {  // 64 columns at a time
                        uint32_t a[2][32];
                        tmem_ld32(trow + (uint32_t)(b * 128 + 64 * h), a[0]);
                        tmem_ld32(trow + (uint32_t)(b * 128 + 64 * h + 32), a[1]);
                        tmem_ld_wait();
                        tmem_ld_dep(a[0]);
                        tmem_ld_dep(a[1]);
                        if (h == 1) {
                            tc_fence_before();
                            mbar_arrive(&sh.acc_empty[b]);
                        }
#pragma unroll
                        for (int q = 0; q < 2; ++q)
#pragma unroll
                            for (int e = 0; e < 32; e += 2) {
                                // packed float32 pairs: the same per-element rounding as fmaf
                                const float2 lv = *reinterpret_cast<const float2*>(live + c * PT_CH + 64 * h + 32 * q + e);
                                const float2 v = __ffma2_rn(make_float2(__uint_as_float(a[q][e]), __uint_as_float(a[q][e + 1])),
                                                            sl2e2, lv);
                                x[q][e] = v.x;
                                x[q][e + 1] = v.y;
                                cm = fmax3f(cm, v.x, v.y);
                            }
                        const float mn = fmaxf(m, cm);
                        if (mn != NEG) {
                            if (mn != m) {
                                l *= (double)fast_exp2(m - mn);  // 0 while m = -inf
                                m = mn;
                            }
#pragma unroll
                            for (int k = 0; k < 8; ++k) part[k] = 0.f;
                            const float2 nm2 = make_float2(-m, -m);
#pragma unroll
                            for (int q = 0; q < 2; ++q)
#pragma unroll
                                for (int e = 0; e < 32; e += 2) {
                                    const float2 d = __fadd2_rn(make_float2(x[q][e], x[q][e + 1]), nm2);
                                    const float2 pp = __fadd2_rn(make_float2(part[e & 7], part[(e + 1) & 7]),
                                                                 make_float2(fast_exp2(d.x), fast_exp2(d.y)));
                                    part[e & 7] = pp.x;
                                    part[(e + 1) & 7] = pp.y;
                                }
                            l += (double)(((part[0] + part[1]) + (part[2] + part[3])) +
                                          ((part[4] + part[5]) + (part[6] + part[7])));
                        }
                    }
                }
                // the two groups meet: row maximum M and denominator L
                sh.xm[grp][row] = m;
                sh.xl[grp][row] = l;
                named_bar_sync(2 + quad, 64);
                const float m0 = sh.xm[0][row], m1 = sh.xm[1][row];
                const float M = fmaxf(m0, m1);
                const double L = (m0 == NEG ? 0.0 : sh.xl[0][row] * (double)fast_exp2(m0 - M)) +
                                 (m1 == NEG ? 0.0 : sh.xl[1][row] * (double)fast_exp2(m1 - M));
                const float inv = valid && L > 0.0 ? (float)(1.0 / L) : 0.f;
                const float2 inv2 = make_float2(inv, inv), nM2 = make_float2(-M, -M);
                named_bar_sync(2 + quad, 64);  // both read before the next tile overwrites
                // pass 2: normalised probabilities, column sums over the warp's 32 rows
                for (int c = 0; c < nch; ++c, ++G) {
                    if ((G & 1) != grp) continue;
                    const int b = G % PT_NB;
                    wait_acc(b, G);
                    float* cs = colsum + quad * nch * PT_CH + c * PT_CH;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t a[32];
                        tmem_ld32(trow + (uint32_t)(b * 128 + 32 * q), a);
                        tmem_ld_wait();
                        tmem_ld_dep(a);
                        if (q == 3) {
                            tc_fence_before();
                            mbar_arrive(&sh.acc_empty[b]);
                        }
                        float v[32];
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            // packed float32 pairs: the same per-element roundings as fmaf, - and *
                            const float2 lv = *reinterpret_cast<const float2*>(live + c * PT_CH + 32 * q + e);
                            const float2 xx =
                                __fadd2_rn(__ffma2_rn(make_float2(__uint_as_float(a[e]), __uint_as_float(a[e + 1])),
                                                      sl2e2, lv),
                                           nM2);
                            const float2 pe = __fmul2_rn(make_float2(fast_exp2(xx.x), fast_exp2(xx.y)), inv2);
                            v[e] = valid ? pe.x : 0.f;  // rows past the cluster add nothing
                            v[e + 1] = valid ? pe.y : 0.f;
                        }
                        cs[32 * q + lane] += transpose_sum32(v, lane);
                    }
                }
            }
            // importance row and its bound
            dmax = warp_max(dmax);
            if (lane == 0) sh.sdmax[warp - 2] = dmax;
            named_bar_sync(1, 256);
            const float invn = 1.0f / (float)nr;
            for (int mm = et; mm < NK; mm += 256) {
                const int stride = nch * PT_CH;
                const float s = ((colsum[mm] + colsum[stride + mm]) + colsum[2 * stride + mm]) + colsum[3 * stride + mm];
                Irow[mm] = s * invn;
            }
            if (et == 0) {
                float qm = 0.f;
                for (int w = 0; w < 8; ++w) qm = fmaxf(qm, sh.sdmax[w]);
                // logit error (natural log units) of the kappa model; exp2 roundings
                // (numerator and denominator); the float32 row-sum partials (8 x 8
                // terms per 64 columns, relative error <= 10 2^-24; 12 counted) and the
                // float32 column sums
                // (+ products and partial sums that the tensor core may flush below
                // 2^-126: at most 2D of them, 2^-118 in all, times the scale)
                double delta = (double)delta_scale * qm * ckmax[bh] + 0x1p-118;
                if (size_prior) delta += 0.6931471805599453 * 5.9604644775390625e-8 * log2((double)N + 1.0);
                const double rr = expm1(2.0 * delta) + 4.0 * 4.76837158203125e-7 +
                                  (12.0 + 16.0 + nr / 64.0) * 5.9604644775390625e-8;
                rho[it] = (float)(rr * 1.001);
            }
        }
        if (failed) *abort = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, PT_TMEM_COLS);
    }
    if (threadIdx.x == 0 && sh.abort) set_status(status, PARK_ERR_TIMEOUT);
}

size_t pama_tc_smem_bytes(int NK) {
    const int nch = (NK + PT_CH - 1) / PT_CH;
    return (size_t)6 * PT_BLK + (size_t)nch * PT_CH * 4 * 5 + 1024;
}

int launch_pama_tc(const void* Qg, int BH, int N, int NQ, int NK, const int32_t* q_perm, const int32_t* q_off,
                   const void* CK, const int32_t* k_off, const float* qnorm, int size_prior, float* importance,
                   float* rho, const float* ckmax, int32_t* status, int num_sms, cudaStream_t st) {
    const int D = 128;
    CUtensorMap mQ, mC;
    PARK_CHECK(make_tma_map_bf16(&mQ, Qg, (uint64_t)BH * N, 128, PT_ROWS));
    PARK_CHECK(make_tma_map_bf16(&mC, CK, (uint64_t)BH * NK, 128, PT_CH));
    const size_t sm = pama_tc_smem_bytes(NK);
    if (sm > 227 * 1024) return PARK_ERR_UNSUPPORTED;
    cudaFuncSetAttribute(k_pama_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    const float scale = 1.0f / sqrtf((float)D);
    const float sl2e = scale * 1.4426950408889634f;
    // |logit~ - logit| <= s (kappa 2^-24 + 2^-23) ||q|| max||c|| (kappa = 2 D / 16 = 16 at D = 128)
    const double kappa = 2.0 * D / 16.0;
    const float delta_scale =
        (float)((1.0 / sqrt((double)D)) * (kappa * 5.9604644775390625e-8 + 1.1920928955078125e-7) * 1.01);
    ::park::prof_begin(st);
    k_pama_tc<<<num_sms, 320, sm, st>>>(mQ, mC, q_perm, q_off, k_off, qnorm, ckmax, N, NQ, NK, BH, sl2e, delta_scale,
                                        size_prior, importance, rho, status, wait_limit_ns());
    PARK_TRY_LAUNCH("k_pama_tc", st);
    return PARK_OK;
}

}  // namespace park
