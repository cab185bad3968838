// Block-sparse attention on the 5th-generation tensor cores (tcgen05 + TMEM +
// TMA), bf16 inputs, D = 128.  With SIP block weights (AB-Attention's inverse
// inclusion probabilities) the per-column bias of a real key row is log2 of its
// block's weight instead of 0, which weights both Softmax sums.
//
// Work items are 128-row query tiles.  Q is gathered into an item-major image
// (item i owns rows 128 i .. 128 i + 127).  Exact query-tile packing: the last
// tile of a query cluster with several tiles (a guest) may share the single tile
// of a smaller cluster (its host); the item's key list is then the union of both
// kept sets, and each row masks the key clusters its own cluster does not keep
// (two column-bias vectors per key tile: own rows, guest rows).  K and V are gathered into cluster order with every key
// cluster padded to a multiple of 8 rows (zero rows), so a kept key cluster is
// a run of whole 8-row groups.  For a query cluster, its kept key clusters are
// concatenated (padded sizes) into one virtual key sequence that is cut into
// full 128-row tiles: clusters smaller than a tile share a tile (the
// gather-into-full-tiles idea of the AB-Attention article).  Padded K and V
// are stored in global memory as the byte image of the shared-memory tiles
// (8-row groups of 2048 bytes: both 64-column halves, 128-byte swizzled), so
// the part of a kept cluster that falls in a tile arrives with one bulk copy
// for K and one for V; pad rows and groups past the end are masked.
//
// One CTA per SM (persistent, work items round-robin), 11 warps:
//   warp 0     producer: Q tile (128 x 128, TMA) per item and each key tile's K
//              (bulk copies, one per kept-cluster piece) into a 3-stage ring;
//   warp 10    producer: each key tile's V into a 2-stage ring, with the
//              per-tile column biases (0, log2 w, or -inf for masked rows) for
//              the own and the guest rows.  The
//              two producers walk the same segment cursor, so K of tile j+3
//              may arrive while V of tile j is still in use;
//   warp 1     TMEM owner and MMA issuer (one thread): S_j = Q K_j^T into TMEM
//              buffer j%2 (128 x 128 fp32), and for each column half h of the
//              tile O_h += P_j,h V_j,h (K = 64) into that half's own TMEM
//              accumulator (128 x 128 fp32), issued as soon as the half's P is
//              in TMEM, in the order S0 S1 PV0 S2 PV1 S3 ...; tcgen05 MMAs of
//              one thread run in issue order, so S_{j+2} overwrites buffer j%2
//              only after PV_j has read P_j from it.
//   warps 2-9  Softmax, two threads per query row (= TMEM lane; warps w and
//              w+4 share a lane quadrant), each owning 64 of a tile's 128
//              columns, with packed float32 pair arithmetic.  Online Softmax in
//              the log2 domain with a lazily updated reference max (the half's
//              O is rescaled in TMEM only when its max grows by more than 2^8).
//              Each half keeps its own reference, row sum and O accumulator, so
//              the two threads of a row never wait for each other within an
//              item.  P_j of a half is written as bf16 pairs over the first 32
//              of the half's own 64 columns of S_j's TMEM buffer (the A operand
//              of that half's PV MMA).  At the end of the item the two halves
//              meet once: O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / (l_0 2^(m_0 - M)
//              + l_1 2^(m_1 - M)) with M = max(m_0, m_1), and each thread writes
//              its half of the O row in original token order.
// Every wait is time-bounded; a timeout sets PARK_ERR_TIMEOUT in the status
// word, the roles leave their loops, outstanding copies and MMAs are waited
// for (bounded) and TMEM is freed before the CTA exits.  Decisions that guard
// warp-collective operations (tcgen05.ld/st, shuffles) are warp-uniform.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"
#include "sm100.cuh"

namespace park {

using namespace sm100;

namespace {
constexpr int TC_ROWS = 128;            // query rows and key rows per tile
constexpr int TC_BLK = 16384;           // 128 rows x 128 bytes
constexpr int TC_KST = 3;  // K ring stages
constexpr int TC_VST = 2;  // V ring stages (with the column bias)
constexpr uint32_t TC_TMEM_COLS = 512;  // S0 [0,128), S1 [128,256), O_0 [256,384), O_1 [384,512)
constexpr float kLog2eT = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may reach 2^8 before O is rescaled

struct TcSmem {
    uint64_t q_full, q_empty, k_full[TC_KST], k_empty[TC_KST], v_full[TC_VST], v_empty[TC_VST], s_full[2],
        p_full[2][2], pv_done[2], o_empty, final_bar;  // p_full[column half][S buffer]
    uint32_t tmem_base;
    int abort;
    alignas(16) float bias[TC_VST][2][TC_ROWS];  // per stage, for the item's own rows [0] and its guest rows [1]:
                                                 // the logit term of a real key row, -inf for a pad row, a row
                                                 // past the end or a key cluster those query rows do not keep
    float xm[2][2][TC_ROWS];             // [item parity][column half][row]: the half's reference max
    float xl[2][2][TC_ROWS];             // [item parity][column half][row]: the half's row sum
};
}  // namespace

__device__ __forceinline__ float bits_f(uint32_t u) { return __uint_as_float(u); }
// warp-uniform view of the abort flag
__device__ __forceinline__ bool warp_abort(volatile int* abort) { return __any_sync(0xffffffffu, *abort != 0); }
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fast_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __launch_bounds__(352, 1)
    k_sparse_attn_tc(const __grid_constant__ CUtensorMap tmQ, const uint8_t* __restrict__ Kimg,
                     const uint8_t* __restrict__ Vimg, int N, int NQ, int NK, const int32_t* __restrict__ q_perm,
                     const int2* __restrict__ segs, const float* __restrict__ segwA,
                     const float* __restrict__ segwB, const int32_t* __restrict__ kv_nseg,
                     const int32_t* __restrict__ kv_pre, const int32_t* __restrict__ kv_len,
                     const WorkItem* __restrict__ items, const int32_t* __restrict__ item_count,
                     uint16_t* __restrict__ O, float sl2e, int32_t* __restrict__ status, uint64_t wait_ns) {
    extern __shared__ __align__(1024) uint8_t dsmem_raw[];
    __shared__ TcSmem sh;
    // 1024-byte aligned operand area: Q | K0 K1 | V0 V1 (each 32 KB)
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Qs = base;
    uint8_t* Ks = base + 2 * TC_BLK;
    uint8_t* Vs = Ks + 2 * TC_KST * TC_BLK;  // TC_VST stages follow

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort = &sh.abort;
    if (threadIdx.x == 0) {
        mbar_init(&sh.q_full, 1);
        mbar_init(&sh.q_empty, 1);
        for (int s = 0; s < TC_KST; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], 1);
        }
        for (int s = 0; s < TC_VST; ++s) {
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.s_full[s], 1);
            mbar_init(&sh.p_full[0][s], 128);
            mbar_init(&sh.p_full[1][s], 128);
            mbar_init(&sh.pv_done[s], 1);
        }
        mbar_init(&sh.o_empty, 256);
        mbar_init(&sh.final_bar, 1);
        sh.abort = 0;
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) tma_prefetch_desc(&tmQ);
    if (warp == 1) {
        tmem_alloc(&sh.tmem_base, TC_TMEM_COLS);
        tmem_relinquish();
    }
    // K/V stages start as zeros: groups that are never loaded must hold finite values
    for (int i = threadIdx.x; i < 2 * (TC_KST + TC_VST) * TC_BLK / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(Ks)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int n_items = *item_count;
    const uint32_t idS = idesc_bf16(128, 128, 0, 0);   // S = Q K^T: both K-major
    const uint32_t idPV = idesc_bf16(128, 128, 0, 1);  // O += P V: P K-major (TMEM), V MN-major

    if (warp == 0 || warp == 10) {
        // ------------------------------------------------------------ producers
        // Warp 0: Q and K (3-stage ring); warp 10: V and the column bias (2-stage
        // ring).  Both walk the same items and tiles with the same segment cursor,
        // so a V stage that waits for its PV never holds up the K loads.
        const bool isK = warp == 0;
        int T = 0, I = 0;
        int k_last[TC_KST], v_last[TC_VST];
        for (int q = 0; q < TC_KST; ++q) k_last[q] = -1;
        for (int q = 0; q < TC_VST; ++q) v_last[q] = -1;
        int q_pending = 0, q_parity = 0;
        for (int it = blockIdx.x; it < n_items && !warp_abort(abort); it += gridDim.x) {
            const WorkItem wi = items[it];
            const int L = kv_len[(size_t)wi.bh * NQ + wi.r];
            const int nkt = (L + TC_ROWS - 1) / TC_ROWS;
            if (nkt == 0) continue;
            const size_t slot = (size_t)wi.bh * NQ + wi.r;  // the item's key list, NK entries per slot
            const int nk = kv_nseg[slot];
            const int32_t* pre = kv_pre + slot * NK;
            const int2* segs_item = segs + slot * NK;
            const float* segwA_item = segwA + slot * NK;
            const float* segwB_item = segwB + slot * NK;
            if (isK && lane == 0) {
                bool ok = I == 0 || mbar_wait(&sh.q_empty, (I - 1) & 1, abort, wait_ns);
                if (ok) {
                    mbar_arrive_expect_tx(&sh.q_full, 2 * TC_BLK);
                    const int y = it * TC_ROWS;  // the item's rows in the item-major Q image
                    tma_load_2d(Qs, &tmQ, &sh.q_full, 0, y);
                    tma_load_2d(Qs + TC_BLK, &tmQ, &sh.q_full, 64, y);
                    q_pending = 1;
                    q_parity = I & 1;
                }
            }
            __syncwarp();
            if (warp_abort(abort)) break;
            // Segment cursor: lane l holds entry seg0 + l of the item's kept
            // segments (prefix of padded sizes, first padded row, size); a tile
            // spans at most 17 segments (each is >= 8 rows), so 32 lanes cover it.
            int seg0 = 0, p_l = 0x7fffffff, src_l = 0, sz_l = 0;
            // additive logit terms of the segment for the own and the guest rows (log2
            // of the block weight, 0 without weights, -inf where those rows do not keep it)
            float lwA_l = 0.f, lwB_l = 0.f;
            auto load_entries = [&](int s0) {
                const int idx = s0 + lane;
                if (idx < nk) {
                    p_l = pre[idx];
                    const int2 e = segs_item[idx];
                    src_l = e.x;
                    sz_l = e.y;
                    lwA_l = segwA_item[idx];
                    lwB_l = segwB_item[idx];
                } else {
                    p_l = 0x7fffffff;
                    src_l = 0;
                    sz_l = 0;
                    lwA_l = lwB_l = 0.f;
                }
            };
            load_entries(0);
            bool ok = true;
            for (int j = 0; j < nkt && ok; ++j) {
                const int stg = T % TC_VST, round = T / TC_VST;
                int nvalid = 0;                // real key rows of group `lane` (lanes 0..15; V warp)
                float lwvA = 0.f, lwvB = 0.f;  // and the logit terms of its segment
#pragma unroll 4
                for (int g = 0; g < 16 && !isK; ++g) {
                    const int vg = j * TC_ROWS + 8 * g;
                    const unsigned bal = __ballot_sync(0xffffffffu, p_l <= vg);
                    const int idx = (__popc(bal) - 1) & 31;
                    const int pp = __shfl_sync(0xffffffffu, p_l, idx);
                    const int sz = __shfl_sync(0xffffffffu, sz_l, idx);
                    const float lwa = __shfl_sync(0xffffffffu, lwA_l, idx);
                    const float lwb = __shfl_sync(0xffffffffu, lwB_l, idx);
                    if (lane == g && vg < L) {
                        int nv = sz - (vg - pp);
                        nvalid = nv < 0 ? 0 : (nv > 8 ? 8 : nv);
                        lwvA = lwa;
                        lwvB = lwb;
                    }
                }
                // this lane's segment (seg0 + lane) as one piece of whole 8-row groups of the tile
                const int t0 = j * TC_ROWS, t1 = min(t0 + TC_ROWS, L);
                int pc_start = 0, pc_groups = 0, pc_src = 0;
                if (p_l < t1) {
                    const int seg_end = p_l + ((sz_l + 7) & ~7);
                    const int a = max(p_l, t0), b = min(seg_end, t1);
                    if (b > a) {
                        pc_start = a - t0;
                        pc_groups = (b - a) >> 3;
                        pc_src = src_l + (a - p_l);
                    }
                }
                const size_t src_off = (size_t)(pc_src >> 3) * 2048;
                const uint32_t bytes = (uint32_t)pc_groups * 2048u;
                const uint32_t tile_bytes = (uint32_t)(t1 - t0) * 256u;
                {  // advance the cursor and prefetch the next tile's entries
                    const int vn = (j + 1) * TC_ROWS;
                    if (vn < L) {
                        const unsigned bal = __ballot_sync(0xffffffffu, p_l <= vn);
                        seg0 += __popc(bal) - 1;
                        load_entries(seg0);
                    }
                }
                if (isK) {
                    // K of tile j: stage free once S_{j-3} has completed
                    const int ks = T % TC_KST, kround = T / TC_KST;
                    bool w = true;
                    if (lane == 0 && kround > 0) w = mbar_wait(&sh.k_empty[ks], (kround - 1) & 1, abort, wait_ns);
                    if (__shfl_sync(0xffffffffu, w ? 1 : 0, 0) == 0 || warp_abort(abort)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) mbar_arrive_expect_tx(&sh.k_full[ks], tile_bytes);
                    __syncwarp();
                    if (pc_groups > 0)
                        bulk_load(Ks + ks * 2 * TC_BLK + (pc_start >> 3) * 2048, Kimg + src_off, bytes,
                                  &sh.k_full[ks]);
                    k_last[ks] = kround & 1;
                } else {
                    // V of tile j and its column bias: free once PV_{j-2} has completed
                    bool w = true;
                    if (lane == 0 && round > 0) w = mbar_wait(&sh.v_empty[stg], (round - 1) & 1, abort, wait_ns);
                    if (__shfl_sync(0xffffffffu, w ? 1 : 0, 0) == 0 || warp_abort(abort)) {
                        ok = false;
                        break;
                    }
                    if (lane < 16) {
                        const float NI = __int_as_float(0xff800000);
#pragma unroll
                        for (int v = 0; v < 2; ++v) {
                            const float lwv = v == 0 ? lwvA : lwvB;
                            float4* bp = reinterpret_cast<float4*>(&sh.bias[stg][v][8 * lane]);
                            bp[0] = make_float4(nvalid > 0 ? lwv : NI, nvalid > 1 ? lwv : NI, nvalid > 2 ? lwv : NI,
                                                nvalid > 3 ? lwv : NI);
                            bp[1] = make_float4(nvalid > 4 ? lwv : NI, nvalid > 5 ? lwv : NI, nvalid > 6 ? lwv : NI,
                                                nvalid > 7 ? lwv : NI);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive_expect_tx(&sh.v_full[stg], tile_bytes);
                    __syncwarp();
                    if (pc_groups > 0)
                        bulk_load(Vs + stg * 2 * TC_BLK + (pc_start >> 3) * 2048, Vimg + src_off, bytes,
                                  &sh.v_full[stg]);
                    v_last[stg] = round & 1;
                }
                ++T;
            }
            if (!ok) break;
            ++I;
        }
        // drain: copies still in flight complete before the CTA may exit
        if (lane == 0) {
            int dummy = 0;
            for (int s = 0; s < TC_KST; ++s)
                if (k_last[s] >= 0) mbar_wait(&sh.k_full[s], k_last[s], &dummy, 100000000ull);
            for (int s = 0; s < TC_VST; ++s)
                if (v_last[s] >= 0) mbar_wait(&sh.v_full[s], v_last[s], &dummy, 100000000ull);
            if (q_pending) mbar_wait(&sh.q_full, q_parity, &dummy, 100000000ull);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int G = 0, I = 0;
            const uint32_t qa = smem_u32(Qs);
            auto issue_S = [&](int g) -> bool {
                const int b = g & 1, ks = g % TC_KST;
                // buffer b is free: its last reader, PV_{g-2}, was issued before this MMA
                if (!mbar_wait(&sh.k_full[ks], (g / TC_KST) & 1, abort, wait_ns)) return false;
                tc_fence_after();
                const uint32_t ka = smem_u32(Ks + ks * 2 * TC_BLK);
                const uint32_t d = tmem + (uint32_t)(b * 128);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t qoff = (uint32_t)((kk >> 2) * TC_BLK + (kk & 3) * 32);
                    const uint32_t koff = (uint32_t)((kk >> 2) * 1024 + (kk & 3) * 32);
                    umma_bf16(d, sdesc_sw128(qa + qoff, 16, 1024), sdesc_sw128(ka + koff, 16, 2048), idS, kk > 0);
                }
                umma_commit(&sh.s_full[b]);
                umma_commit(&sh.k_empty[ks]);
                return true;
            };
            for (int it = blockIdx.x; it < n_items && !*abort; it += gridDim.x) {
                const WorkItem wi = items[it];
                const int L = kv_len[(size_t)wi.bh * NQ + wi.r];
                const int nkt = (L + TC_ROWS - 1) / TC_ROWS;
                if (nkt == 0) continue;
                if (!mbar_wait(&sh.q_full, I & 1, abort, wait_ns)) break;
                tc_fence_after();
                bool ok = issue_S(G) && (nkt < 2 || issue_S(G + 1));
                for (int j = 0; j < nkt && ok; ++j) {
                    const int g = G + j, b = g & 1, ph = (g >> 1) & 1, vs = g % TC_VST;
                    if ((j == 0 && I > 0 && !mbar_wait(&sh.o_empty, (I - 1) & 1, abort, wait_ns)) ||
                        !mbar_wait(&sh.v_full[vs], (g / TC_VST) & 1, abort, wait_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t va = smem_u32(Vs + vs * 2 * TC_BLK);
                    // each column half's keys (V rows 64 h .. 64 h + 63) into its own O_h, as
                    // soon as that half's P is in TMEM (columns 64 h .. 64 h + 31 of buffer b)
                    for (int h = 0; h < 2 && ok; ++h) {
                        if (!mbar_wait(&sh.p_full[h][b], ph, abort, wait_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16_ts(tmem + 256u + 128u * h, tmem + (uint32_t)(b * 128 + 64 * h + 8 * kk),
                                         sdesc_sw128(va + (uint32_t)(4 * h + kk) * 4096, 1024, 2048), idPV,
                                         (j > 0 || kk > 0));
                    }
                    if (!ok) break;
                    umma_commit(&sh.pv_done[b]);
                    umma_commit(&sh.v_empty[vs]);
                    if (j + 2 < nkt && !issue_S(g + 2)) ok = false;
                }
                if (!ok) break;
                umma_commit(&sh.q_empty);
                G += nkt;
                ++I;
            }
            // every MMA issued so far has completed before TMEM is released
            umma_commit(&sh.final_bar);
            int dummy = 0;
            mbar_wait(&sh.final_bar, 0, &dummy, 100000000ull);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int quad = warp & 3, hc = (warp - 2) >> 2;  // lane quadrant, column half
        const int row = 32 * quad + lane;
        const uint32_t trow = tmem + ((uint32_t)(32 * quad) << 16);
        const int pair_bar = 1 + quad;  // named barrier of warps w and w+4 (64 threads)
        const uint32_t o_col = 256u + 128u * (uint32_t)hc;  // this half's O accumulator
        const float2 sl2e2 = make_float2(sl2e, sl2e);
        int G = 0, I = 0;
        // Waits are decided per warp (tcgen05.ld/st and shuffles are warp-collective).
        // The two warps of a pair pass their named barrier (once per item) the same number
        // of times whatever happens: after a failed wait a warp skips every later wait and
        // all tensor-memory work but still walks the items and meets its barriers.
        bool failed = false;
        auto wwait = [&](uint64_t* bar, uint32_t parity) {
            if (!failed) failed = !__all_sync(0xffffffffu, mbar_wait(bar, parity, abort, wait_ns));
            return !failed;
        };
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const WorkItem wi = items[it];
            const int L = kv_len[(size_t)wi.bh * NQ + wi.r];
            const int nkt = (L + TC_ROWS - 1) / TC_ROWS;
            if (nkt == 0) continue;
            float m_ref = __int_as_float(0xff800000);
            float2 l2 = make_float2(0.f, 0.f);  // partial row sums of the even and odd columns
            for (int j = 0; j < nkt; ++j) {
                const int g = G + j, b = g & 1, ph = (g >> 1) & 1, vs = g % TC_VST;
                const bool live = wwait(&sh.s_full[b], ph) && wwait(&sh.v_full[vs], (g / TC_VST) & 1);
                uint32_t s[2][32];
                float tm[2] = {__int_as_float(0xff800000), __int_as_float(0xff800000)};
                if (live) {
                    tc_fence_after();
                    tmem_ld32(trow + (uint32_t)(b * 128 + 64 * hc), s[0]);
                    tmem_ld32(trow + (uint32_t)(b * 128 + 64 * hc + 32), s[1]);
                    tmem_ld_wait();
                    tmem_ld_dep(s[0]);
                    tmem_ld_dep(s[1]);
                    // the guest rows of a packed item [rows, rows + g_rows) keep their own key clusters
                    const float4* bz = reinterpret_cast<const float4*>(sh.bias[vs][row < wi.rows ? 0 : 1] + 64 * hc);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            // packed float32 pairs: one FMA instruction per two elements
                            const float4 bb = bz[c * 8 + q];
                            const float2 x01 = __ffma2_rn(make_float2(bits_f(s[c][4 * q]), bits_f(s[c][4 * q + 1])),
                                                          sl2e2, make_float2(bb.x, bb.y));
                            const float2 x23 = __ffma2_rn(
                                make_float2(bits_f(s[c][4 * q + 2]), bits_f(s[c][4 * q + 3])), sl2e2,
                                make_float2(bb.z, bb.w));
                            s[c][4 * q + 0] = __float_as_uint(x01.x);
                            s[c][4 * q + 1] = __float_as_uint(x01.y);
                            s[c][4 * q + 2] = __float_as_uint(x23.x);
                            s[c][4 * q + 3] = __float_as_uint(x23.y);
                            tm[0] = fmax3f(tm[0], x01.x, x01.y);
                            tm[1] = fmax3f(tm[1], x23.x, x23.y);
                        }
                    }
                }
                if (!live) continue;
                const float tmax = fmaxf(tm[0], tm[1]);  // this half's tile max
                if (j == 0) {
                    m_ref = tmax;
                } else if (__any_sync(0xffffffffu, tmax > m_ref + kRescaleThreshold)) {
                    // decided per warp; rows that keep their reference get alpha = 1.  O_h
                    // must hold PV_{j-1}.
                    if (!wwait(&sh.pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1)) continue;
                    tc_fence_after();
                    const float m_new = tmax > m_ref + kRescaleThreshold ? tmax : m_ref;
                    const float alpha = m_new == m_ref ? 1.f : fast_ex2(m_ref - m_new);  // (m_ref may be -inf)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tmem_ld32(trow + o_col + (uint32_t)(32 * c), o);
                        tmem_ld_wait();
                        tmem_ld_dep(o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(bits_f(o[e]) * alpha);
                        tmem_st32(trow + o_col + (uint32_t)(32 * c), o);
                    }
                    tmem_st_wait();
                    l2.x *= alpha;
                    l2.y *= alpha;
                    m_ref = m_new;
                }
                // P (bf16 pairs) over the first 32 of this half's own 64 columns of buffer b
                // (S values this thread has already read)
                uint32_t pk[32];
                // a row that has met only masked keys so far (the guest rows of a packed item
                // can) keeps m_ref = -inf: its P is 0, and the first real maximum rescales O by 0
                const float mr = m_ref == __int_as_float(0xff800000) ? 0.f : m_ref;
                const float2 nm2 = make_float2(-mr, -mr);
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 d = __fadd2_rn(make_float2(bits_f(s[c][2 * e]), bits_f(s[c][2 * e + 1])), nm2);
                        const float p0 = fast_ex2(d.x);
                        const float p1 = fast_ex2(d.y);
                        l2 = __fadd2_rn(l2, make_float2(p0, p1));
                        __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                        pk[16 * c + e] = *reinterpret_cast<uint32_t*>(&h);
                    }
                tmem_st32(trow + (uint32_t)(b * 128 + 64 * hc), pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&sh.p_full[hc][b]);
            }
            // epilogue: the two halves meet once per item.  O = (O_0 a_0 + O_1 a_1) / l with
            // a_h = 2^(m_h - M), M = max(m_0, m_1), l = l_0 a_0 + l_1 a_1; original token order;
            // each thread writes its 64 columns.  The shared slots alternate by item, so the
            // partner overwrites them only after the next item's barrier, which this thread
            // reaches after reading them.
            sh.xm[I & 1][hc][row] = m_ref;
            sh.xl[I & 1][hc][row] = l2.x + l2.y;
            named_bar_sync(pair_bar, 64);
            const float m0 = sh.xm[I & 1][0][row], m1 = sh.xm[I & 1][1][row];
            const float M = fmaxf(m0, m1);
            const float a0 = m0 == __int_as_float(0xff800000) ? 0.f : fast_ex2(m0 - M);
            const float a1 = m1 == __int_as_float(0xff800000) ? 0.f : fast_ex2(m1 - M);
            const float lt = sh.xl[I & 1][0][row] * a0 + sh.xl[I & 1][1][row] * a1;
            const int gl = G + nkt - 1;
            G += nkt;
            ++I;
            if (!wwait(&sh.pv_done[gl & 1], (gl >> 1) & 1)) continue;
            tc_fence_after();
            const int grow = row - wi.rows;  // row of the guest part, if any
            const bool wr = row < wi.rows || grow < wi.g_rows;
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            const int tok = !wr ? 0
                                : (row < wi.rows ? q_perm[(size_t)wi.bh * N + wi.q_start + row]
                                                 : q_perm[(size_t)wi.bh * N + wi.g_start + grow]);
            uint4* dst = reinterpret_cast<uint4*>(O + ((size_t)wi.bh * N + tok) * 128 + 64 * hc);
            const float s0 = a0 * inv, s1 = a1 * inv;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t o0[32], o1[32];
                tmem_ld32(trow + 256u + (uint32_t)(64 * hc + 32 * c), o0);
                tmem_ld32(trow + 384u + (uint32_t)(64 * hc + 32 * c), o1);
                tmem_ld_wait();
                tmem_ld_dep(o0);
                tmem_ld_dep(o1);
                if (c == 1) {
                    tc_fence_before();
                    mbar_arrive(&sh.o_empty);
                }
                if (wr) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = 8 * q + 2 * e;
                            __nv_bfloat162 h =
                                __floats2bfloat162_rn(fmaf(bits_f(o0[k]), s0, bits_f(o1[k]) * s1),
                                                      fmaf(bits_f(o0[k + 1]), s0, bits_f(o1[k + 1]) * s1));
                            w4[e] = *reinterpret_cast<uint32_t*>(&h);
                        }
                        dst[c * 4 + q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TC_TMEM_COLS);
    }
    if (threadIdx.x == 0 && sh.abort) set_status(status, PARK_ERR_TIMEOUT);
}

// ---------------------------------------------------------------- host side
namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_encode_mu;
}  // namespace

// 2-D bf16 tensor [rows][cols] (row-major), boxes of 64 columns x box_rows,
// 128-byte swizzle.  The driver entry point is looked up once.
int make_tma_map_bf16(CUtensorMap* map, const void* ptr, uint64_t rows, uint32_t cols, uint32_t box_rows) {
    {
        std::lock_guard<std::mutex> lk(g_encode_mu);
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn) {
                cudaGetLastError();
                return PARK_ERR_CUDA;
            }
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
    }
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PARK_OK : PARK_ERR_CUDA;
}

size_t attn_tc_smem_bytes() { return (size_t)(2 + 2 * TC_KST + 2 * TC_VST) * TC_BLK + 1024; }  // Q, K and V rings

int launch_sparse_attn_tc(const void* Qimg, size_t item_cap, const void* Kpad, const void* Vpad, int BH, int N, int Npad,
                          int NQ, int NK, const int32_t* q_perm, const int2* segs, const float* segwA,
                          const float* segwB, const int32_t* kv_nseg, const int32_t* kv_pre, const int32_t* kv_len,
                          const WorkItem* items, const int32_t* item_count, void* O, int32_t* status, int num_sms,
                          cudaStream_t st) {
    CUtensorMap mQ;
    PARK_CHECK(make_tma_map_bf16(&mQ, Qimg, (uint64_t)item_cap * TC_ROWS, 128, 128));
    const size_t sm = attn_tc_smem_bytes();
    cudaFuncSetAttribute(k_sparse_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    const float sl2e = (1.0f / sqrtf(128.f)) * kLog2eT;
    ::park::prof_begin(st);
    k_sparse_attn_tc<<<num_sms, 352, sm, st>>>(mQ, (const uint8_t*)Kpad, (const uint8_t*)Vpad, N, NQ, NK, q_perm,
                                                segs, segwA, segwB, kv_nseg, kv_pre, kv_len, items, item_count,
                                                (uint16_t*)O,
                                                sl2e, status, wait_limit_ns());
    PARK_TRY_LAUNCH("k_sparse_attn_tc", st);
    return PARK_OK;
}

}  // namespace park
