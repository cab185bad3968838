// K-means assign step on the 5th-generation tensor cores (tcgen05 + TMEM +
// TMA), bf16 inputs, D = 128.
//
// Scores s~_k = bias_k - 2 x . w_k for every (row, centroid) come from one GEMM:
// rows of X (256-row tiles, TMA) against the centroid operand W streamed in
// chunks of 128 centroids (TMA, 2-stage ring); each chunk feeds two M = 128
// MMAs (rows 0-127 and 128-255), so every centroid byte read serves 256 rows.  Euclidean (queries): w = c,
// K = 128.  QRKC (keys): w = M c split as bf16 hi | lo, K = 256, with the row
// tile used twice as the A operand ([x, x] . [hi; lo] = x . (hi + lo)).
// Accumulators live in TMEM (two buffers x two row halves of 128 x 128 fp32).
// Eight epilogue warps (warps 2-5: rows 0-127, warps 6-9: rows 128-255; one
// thread per row) track, branch-free, the smallest score of their row, its
// column and the second smallest score, in four independent copies (one per
// 32-column group of every chunk) merged once per tile, and apply the
// certified decision of k_assign.cu: the winner is certified when the
// runner-up is more than 2 beta above it, else the row is listed for a float64
// rescore against every centroid.  The head's float bias is staged in shared
// memory.
//
// One CTA per SM, persistent over row tiles; warp 0 loads, warp 1 owns TMEM
// and issues the MMAs (one thread), warps 2-9 are the epilogue.  Every wait is
// time-bounded (PARK_ERR_TIMEOUT on expiry); epilogue warps never leave their
// loops early (after a failed wait they only skip the waits).
#include "kernels.h"
#include "sm100.cuh"

namespace park {

using namespace sm100;

namespace {
constexpr int AS_ROWS = 256, AS_CH = 128, AS_BLK = 16384;
constexpr uint32_t AS_TMEM_COLS = 512;  // 2 buffers x 2 row halves x 128 columns

struct AsSmem {
    uint64_t x_full, x_empty, w_full[2], w_empty[2], acc_full[2], acc_empty[2], final_bar;
    uint32_t tmem_base;
    int abort;
};

}  // namespace

template <int KW>
__global__ void __launch_bounds__(320, 1)
    k_assign_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int N, int K,
                int BH, const float* __restrict__ bias, int bias_ld, const float* __restrict__ xnorm,
                const float* __restrict__ wmax, const float* __restrict__ bmax, float gamma,
                int32_t* __restrict__ labels, Lists lists, int32_t* __restrict__ status,
                uint64_t wait_ns) {
    constexpr int WB = KW / 64;  // 64-column blocks per centroid chunk
    extern __shared__ __align__(1024) uint8_t dsmem_raw[];
    __shared__ AsSmem sh;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Xs = base;               // row halves x 2 column blocks
    uint8_t* Ws = base + 4 * AS_BLK;  // 2 stages x WB blocks
    float* sbias = reinterpret_cast<float*>(Ws + 2 * WB * AS_BLK);  // [nch * 128] bias of the current head
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort = &sh.abort;
    if (threadIdx.x == 0) {
        mbar_init(&sh.x_full, 1);
        mbar_init(&sh.x_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.w_full[s], 1);
            mbar_init(&sh.w_empty[s], 1);
            mbar_init(&sh.acc_full[s], 1);
            mbar_init(&sh.acc_empty[s], 256);
        }
        mbar_init(&sh.final_bar, 1);
        sh.abort = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(&sh.tmem_base, AS_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int tpr = (N + AS_ROWS - 1) / AS_ROWS;  // row tiles per head
    const int ntiles = tpr * BH;
    const int nch = (K + AS_CH - 1) / AS_CH;
    const uint32_t idS = idesc_bf16(128, 128, 0, 0);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int G = 0, I = 0, w_last[2] = {-1, -1}, x_last = -1;
            for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
                const int bh = t / tpr, r0 = (t - bh * tpr) * AS_ROWS;
                if (I > 0 && !mbar_wait(&sh.x_empty, (I - 1) & 1, abort, wait_ns)) break;
                mbar_arrive_expect_tx(&sh.x_full, 4 * AS_BLK);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    tma_load_2d(Xs + 2 * h * AS_BLK, &tmX, &sh.x_full, 0, bh * N + r0 + 128 * h);
                    tma_load_2d(Xs + (2 * h + 1) * AS_BLK, &tmX, &sh.x_full, 64, bh * N + r0 + 128 * h);
                }
                x_last = I & 1;
                bool ok = true;
                for (int c = 0; c < nch; ++c) {
                    const int s = G & 1, round = G >> 1;
                    if (round > 0 && !mbar_wait(&sh.w_empty[s], (round - 1) & 1, abort, wait_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sh.w_full[s], WB * AS_BLK);
#pragma unroll
                    for (int b = 0; b < WB; ++b)
                        tma_load_2d(Ws + (s * WB + b) * AS_BLK, &tmW, &sh.w_full[s], 64 * b, bh * K + c * AS_CH);
                    w_last[s] = round & 1;
                    ++G;
                }
                if (!ok) break;
                ++I;
            }
            int dummy = 0;
            for (int s = 0; s < 2; ++s)
                if (w_last[s] >= 0) mbar_wait(&sh.w_full[s], w_last[s], &dummy, 100000000ull);
            if (x_last >= 0) mbar_wait(&sh.x_full, x_last, &dummy, 100000000ull);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int G = 0, I = 0;
            const uint32_t xa = smem_u32(Xs);
            for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
                if (!mbar_wait(&sh.x_full, I & 1, abort, wait_ns)) break;
                bool ok = true;
                for (int c = 0; c < nch; ++c) {
                    const int s = G & 1, round = G >> 1;
                    if (!mbar_wait(&sh.w_full[s], round & 1, abort, wait_ns) ||
                        (round > 0 && !mbar_wait(&sh.acc_empty[s], (round - 1) & 1, abort, wait_ns))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t wa = smem_u32(Ws + s * WB * AS_BLK);
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int kk = 0; kk < KW / 16; ++kk) {
                            const int xk = kk & 7;  // the row tile serves both halves of [hi | lo]
                            const uint32_t aoff = (uint32_t)((2 * h + (xk >> 2)) * AS_BLK + (xk & 3) * 32);
                            const uint32_t boff = (uint32_t)((kk >> 2) * AS_BLK + (kk & 3) * 32);
                            umma_bf16(tmem + (uint32_t)((2 * s + h) * 128), sdesc_sw128(xa + aoff, 16, 1024),
                                      sdesc_sw128(wa + boff, 16, 1024), idS, kk > 0);
                        }
                    umma_commit(&sh.acc_full[s]);
                    umma_commit(&sh.w_empty[s]);
                    ++G;
                }
                if (!ok) break;
                umma_commit(&sh.x_empty);
                ++I;
            }
            umma_commit(&sh.final_bar);
            int dummy = 0;
            mbar_wait(&sh.final_bar, 0, &dummy, 100000000ull);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int half = (warp - 2) >> 2;  // row half of the tile
        const int lane_base = 32 * (warp & 3);
        const int row = half * 128 + lane_base + lane;
        const uint32_t trow = tmem + ((uint32_t)lane_base << 16) + (uint32_t)(half * 128);
        const float INF = __int_as_float(0x7f800000);
        bool failed = false;
        int G = 0, cur_bh = -1;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const int bh = t / tpr, r0 = (t - bh * tpr) * AS_ROWS;
            if (bh != cur_bh) {  // stage the head's bias (all epilogue warps take this branch together)
                named_bar_sync(1, 256);
                for (int k = threadIdx.x - 64; k < nch * AS_CH; k += 256) sbias[k] = bias[(size_t)bh * bias_ld + k];
                named_bar_sync(1, 256);
                cur_bh = bh;
            }
            // tracker g covers columns 32 g .. 32 g + 31 of every chunk, in increasing order
            float v0[4] = {INF, INF, INF, INF}, v1[4] = {INF, INF, INF, INF};
            int i0[4] = {0, 0, 0, 0};
            for (int c = 0; c < nch; ++c) {
                const int s = G & 1, round = G >> 1;
                if (!failed) {
                    const bool ok = mbar_wait(&sh.acc_full[s], round & 1, abort, wait_ns);
                    failed = !__all_sync(0xffffffffu, ok);
                }
                tc_fence_after();
#pragma unroll
                for (int gp = 0; gp < 2; ++gp) {  // two 32-column groups at a time
                    uint32_t acc[2][32];
                    tmem_ld32(trow + (uint32_t)(2 * s * 128 + 64 * gp), acc[0]);
                    tmem_ld32(trow + (uint32_t)(2 * s * 128 + 64 * gp + 32), acc[1]);
                    tmem_ld_wait();
                    tmem_ld_dep(acc[0]);
                    tmem_ld_dep(acc[1]);
                    if (gp == 1) {  // the whole chunk is in registers: release the accumulator
                        tc_fence_before();
                        mbar_arrive(&sh.acc_empty[s]);
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {  // two trackers interleave for ILP
                            const int g = 2 * gp + h;
                            const int cb = c * AS_CH + 32 * g + 4 * q;
                            const float4 b4 = *reinterpret_cast<const float4*>(sbias + cb);
                            const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float sc = fmaf(-2.f, __uint_as_float(acc[h][4 * q + e]), bv[e]);
                                v1[g] = fminf(v1[g], fmaxf(v0[g], sc));
                                i0[g] = sc < v0[g] ? cb + e : i0[g];  // strict: the first of equal scores stays
                                v0[g] = fminf(v0[g], sc);
                            }
                        }
                }
                ++G;
            }
            // merge: smallest (v0, column), then the second smallest of everything else
            int w = 0;
#pragma unroll
            for (int g = 1; g < 4; ++g)
                if (v0[g] < v0[w] || (v0[g] == v0[w] && i0[g] < i0[w])) w = g;
            float best = v0[w], second = v1[w];
#pragma unroll
            for (int g = 0; g < 4; ++g)
                if (g != w) second = fminf(second, v0[g]);
            if (r0 + row < N && !failed) {
                const size_t gr = (size_t)bh * N + r0 + row;
                // relative terms (accumulation, split residual, bias rounding) plus two
                // absolute ones for magnitudes below the float32/bf16 normal range: bf16
                // hi/lo parts of M c that flush to zero (< 2^-126 each, summed against
                // |x|: <= 2^-121.5 ||x||) and products or partial sums that the tensor
                // core flushes (< 2^-126 each over 256 terms, doubled: covered by 1e-30)
                const float xn = xnorm[gr];
                const float beta = gamma * xn * wmax[bh] + 4.8e-7f * bmax[bh] + xn * 0x1p-118f + 1e-30f;
                labels[gr] = i0[w];
                if (!(second - best > 2.f * beta)) {
                    const int pos = atomicAdd(lists.counts + bh, 1);
                    lists.full_row[(size_t)bh * N + pos] = (int32_t)gr;
                }
            }
        }
        if (failed) *abort = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, AS_TMEM_COLS);
    }
    if (threadIdx.x == 0 && sh.abort) set_status(status, PARK_ERR_TIMEOUT);
}

int launch_assign_tc(const void* X, int BH, int N, int K, const CentroidOps& ops, const float* xnorm, float gamma,
                     int32_t* labels, Lists lists, int32_t* status, int num_sms, cudaStream_t st) {
    if (ops.kw != 128 && ops.kw != 256) return PARK_ERR_UNSUPPORTED;
    CUtensorMap mX, mW;
    PARK_CHECK(make_tma_map_bf16(&mX, X, (uint64_t)BH * N, 128, 128));
    PARK_CHECK(make_tma_map_bf16(&mW, ops.w, (uint64_t)BH * K, (uint32_t)ops.kw, AS_CH));
    const size_t sm = (size_t)(4 + 2 * (ops.kw / 64)) * AS_BLK + 1024 + (size_t)((K + AS_CH - 1) / AS_CH) * AS_CH * 4;
    if (ops.kw == 128)
        cudaFuncSetAttribute(k_assign_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    else
        cudaFuncSetAttribute(k_assign_tc<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    ::park::prof_begin(st);
    if (ops.kw == 128)
        k_assign_tc<128><<<num_sms, 320, sm, st>>>(mX, mW, N, K, BH, ops.bias32, ops.bias_ld, xnorm, ops.wmax,
                                                   ops.bmax, gamma, labels, lists, status, wait_limit_ns());
    else
        k_assign_tc<256><<<num_sms, 320, sm, st>>>(mX, mW, N, K, BH, ops.bias32, ops.bias_ld, xnorm, ops.wmax,
                                                   ops.bmax, gamma, labels, lists, status, wait_limit_ns());
    PARK_TRY_LAUNCH("k_assign_tc", st);
    return PARK_OK;
}

}  // namespace park
