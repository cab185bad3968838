// Block-sparse attention with two query tiles per CTA sharing every K/V tile
// (tcgen05 + TMEM + TMA, bf16, D = 128).
//
// The work items of the query-tile schedule (128-row query tiles, packed with a
// guest cluster's last tile where that saves key tiles) are grouped in pairs
// that walk one key list together:
//   * two tiles of the same query cluster share its key list as it is;
//   * two single-tile clusters of a head that keep mostly the same key
//     clusters are paired over the union of their kept sets when that costs
//     fewer key-tile loads than running them apart (union at most 1.5 x the
//     mean of the two lists); every row still masks the key clusters its own
//     cluster does not keep (a column bias per key tile for each of the four
//     row groups: first tile's own and guest rows, second tile's own and guest
//     rows), so the result is unchanged;
//   * the rest run alone.
// Each K and V tile is then copied from L2 once for two query tiles, and the
// two tiles' Softmax work runs on separate warps that interleave.
//
// One CTA per SM (persistent, pairs round-robin), 11 warps:
//   warp 0     producer: Q of both tiles (TMA from the item-major image) and
//              each key tile's K (bulk copies, one per kept-cluster piece) into
//              a 2-stage ring;
//   warp 10    producer: each key tile's V and the four column-bias rows into a
//              2-stage ring;
//   warp 1     TMEM owner and MMA issuer (one thread).  TMEM: S_A [0,128),
//              S_B [128,256), O_A [256,384), O_B [384,512).  Order per key tile
//              j: S_A(0) S_B(0), then PV_A(j) S_A(j+1) PV_B(j) S_B(j+1) ...; the
//              MMAs of one thread run in issue order, so S_X(j+1) overwrites
//              P_X(j) only after PV_X(j) has read it;
//   warps 2-5  Softmax of the first tile, warps 6-9 of the second: one thread
//              per query row (= TMEM lane), 128 columns in two passes over
//              TMEM (logits with their bias written back in place and the row
//              maximum; then exponentials, the row sum, and P as bf16 pairs over
//              the first 64 columns of S).  Online Softmax in the log2 domain
//              with a lazily updated reference maximum (O is rescaled in TMEM
//              only when a row maximum grows by more than 2^8).  At the end each
//              thread normalises its O row and writes it in original token order.
// Every wait is time-bounded; a timeout sets PARK_ERR_TIMEOUT, the roles leave
// their loops (the Softmax warps keep walking the items without waiting or
// touching TMEM), outstanding copies and MMAs are waited for (bounded) and TMEM
// is freed before the CTA exits.  Decisions that guard warp-collective
// operations (tcgen05.ld/st, shuffles) are warp-uniform.
#include <climits>

#include "kernels.h"
#include "sm100.cuh"

namespace park {

using namespace sm100;

namespace {
constexpr int PR_ROWS = 128;            // query rows and key rows per tile
constexpr int PR_BLK = 16384;           // 128 rows x 128 bytes
constexpr int PR_KST = 2;               // K ring stages
constexpr int PR_VST = 2;               // V ring stages (with the column biases)
constexpr uint32_t PR_TMEM_COLS = 512;  // S_A, S_B, O_A, O_B
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThr = 8.0f;  // log2 units: P may reach 2^8 before O is rescaled
constexpr int kPairWindow = 16;      // pairing candidates: clusters a - 16 .. a + 16 of a head
constexpr int kPairKeep = 8;         // candidates kept per cluster, best first

struct PrSmem {
    uint64_t q_full, q_empty, k_full[PR_KST], k_empty[PR_KST], v_full[PR_VST], v_empty[PR_VST];
    uint64_t s_full[2], p_full[2], pv_done[2], o_empty[2], final_bar;  // [0]: first tile, [1]: second
    uint32_t tmem_base;
    int abort;
    // per V stage, for the row groups (first tile own / guest, second tile own / guest):
    // the logit term of a real key row, -inf for a pad row, a row past the end or a
    // key cluster those query rows do not keep
    alignas(16) float bias[PR_VST][4][PR_ROWS];
};

__device__ __forceinline__ float pr_bits(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ bool pr_warp_abort(volatile int* abort) { return __any_sync(0xffffffffu, *abort != 0); }
__device__ __forceinline__ float pr_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float pr_max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
}  // namespace

// ---------------------------------------------------------------- pairing
// Candidates of a single-tile query cluster a: the single-tile clusters of its
// head within kPairWindow in cluster order (clusters in nearby order come from
// nearby tokens and keep similar key clusters).  Cost of a pair = key tiles of
// the union of the two kept sets (each with its guest's), accepted when at most
// 1.5 x the mean of the two lists; the kPairKeep cheapest, relative to the two
// lists apart, are kept (ties: lower index).
__global__ __launch_bounds__(256) void k_pair_cand(int NQ, int NK, const uint8_t* __restrict__ mask,
                                                   const int32_t* __restrict__ k_off,
                                                   const int32_t* __restrict__ pack_guest,
                                                   const int32_t* __restrict__ slot_items,
                                                   const int32_t* __restrict__ kv_len, int2* __restrict__ cand,
                                                   int32_t* __restrict__ partner) {
    extern __shared__ __align__(16) int32_t pc_sm[];
    int32_t* pd = pc_sm;                                       // [NK] padded cluster sizes
    uint8_t* ma = reinterpret_cast<uint8_t*>(pc_sm + NK);      // [NK] a's kept set (with its guest's)
    __shared__ int cost[2 * kPairWindow], cidx[2 * kPairWindow];
    const int a = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const size_t hb = (size_t)bh * NQ, sa = hb + a;
    int2* out = cand + sa * kPairKeep;
    if (t == 0) partner[sa] = -1;
    if (slot_items[sa] != 1) {
        if (t < kPairKeep) out[t] = make_int2(INT_MAX, -1);
        return;
    }
    const int32_t* ko = k_off + (size_t)bh * (NK + 1);
    const int ga = pack_guest ? pack_guest[sa] : -1;
    const uint8_t* mA = mask + sa * NK;
    const uint8_t* mG = ga >= 0 ? mask + (hb + ga) * NK : nullptr;
    for (int m = t; m < NK; m += blockDim.x) {
        ma[m] = (uint8_t)(mA[m] | (mG ? mG[m] : 0));
        pd[m] = (ko[m + 1] - ko[m] + 7) & ~7;
    }
    __syncthreads();
    const int Ta = (kv_len[sa] + 127) / 128;
    for (int c = w; c < 2 * kPairWindow; c += 8) {
        const int b = c < kPairWindow ? a - kPairWindow + c : a + 1 + (c - kPairWindow);
        int score = INT_MAX, bi = -1;
        if (b >= 0 && b < NQ && slot_items[hb + b] == 1) {
            const int gb = pack_guest ? pack_guest[hb + b] : -1;
            const uint8_t* mB = mask + (hb + b) * NK;
            const uint8_t* mBg = gb >= 0 ? mask + (hb + gb) * NK : nullptr;
            int u = 0;
            for (int m = lane; m < NK; m += 32)
                if (ma[m] | mB[m] | (mBg ? mBg[m] : 0)) u += pd[m];
            u = warp_sum_int(u);
            const int Tu = (u + 127) / 128, Tb = (kv_len[hb + b] + 127) / 128;
            if (Tu > 0 && 4 * Tu <= 3 * (Ta + Tb)) {
                score = (Tu * 4096) / (Ta + Tb);
                bi = b;
            }
        }
        if (lane == 0) {
            cost[c] = score;
            cidx[c] = bi;
        }
    }
    __syncthreads();
    if (t == 0) {  // the kPairKeep cheapest, ties to the lower index
        for (int k = 0; k < kPairKeep; ++k) {
            int best = -1;
            for (int c = 0; c < 2 * kPairWindow; ++c)
                if (cidx[c] >= 0 && (best < 0 || cost[c] < cost[best] || (cost[c] == cost[best] && cidx[c] < cidx[best])))
                    best = c;
            if (best < 0) {
                out[k] = make_int2(INT_MAX, -1);
            } else {
                out[k] = make_int2(cost[best], cidx[best]);
                cidx[best] = -1;
            }
        }
    }
}

// One CTA per head: its candidate lists are staged in shared memory; thread 0
// takes the clusters in order, each pairing with its cheapest listed
// candidate that is still free.
__global__ __launch_bounds__(256) void k_pair_select(int NQ, const int32_t* __restrict__ slot_items,
                                                     const int2* __restrict__ cand, int32_t* __restrict__ partner) {
    extern __shared__ __align__(16) int32_t ps_sm[];
    int2* cs = reinterpret_cast<int2*>(ps_sm);            // [NQ][kPairKeep]
    int32_t* pt = ps_sm + 2 * NQ * kPairKeep;              // [NQ] partner
    int32_t* one = pt + NQ;                                // [NQ] single-tile flag
    const int bh = blockIdx.x, t = threadIdx.x;
    const size_t hb = (size_t)bh * NQ;
    for (int i = t; i < NQ * kPairKeep; i += blockDim.x) cs[i] = cand[hb * kPairKeep + i];
    for (int r = t; r < NQ; r += blockDim.x) {
        pt[r] = -1;
        one[r] = slot_items[hb + r] == 1;
    }
    __syncthreads();
    if (t == 0) {
        for (int a = 0; a < NQ; ++a) {
            if (!one[a] || pt[a] >= 0) continue;
            for (int k = 0; k < kPairKeep; ++k) {
                const int b = cs[a * kPairKeep + k].y;
                if (b < 0) break;
                if (pt[b] >= 0) continue;
                pt[a] = b;
                pt[b] = a;
                break;
            }
        }
    }
    __syncthreads();
    for (int r = t; r < NQ; r += blockDim.x) partner[hb + r] = pt[r];
}

// Key list of every lead cluster a (one that starts a pair, or runs alone):
// the union, in ascending key-cluster order, of the kept sets of a, its guest,
// and for a pair of two clusters its partner b > a and b's guest; per entry the
// padded prefix, the segment (first padded row, size) and the four row groups'
// logit terms (0 or log2 of the block weight where kept, -inf elsewhere).  A
// cluster with several tiles pairs its own tiles: the second tile's rows are
// own rows too.  Counts the (query tile, key tile) pairs computed.
__global__ __launch_bounds__(256) void k_pair_lists(int NQ, int NK, int Npad, const int32_t* __restrict__ k_off,
                                                    const uint8_t* __restrict__ mask,
                                                    const float* __restrict__ bweight,
                                                    const int32_t* __restrict__ poff,
                                                    const int32_t* __restrict__ pack_guest,
                                                    const int32_t* __restrict__ slot_items,
                                                    const int32_t* __restrict__ partner,
                                                    int32_t* __restrict__ pl_pre, int2* __restrict__ pl_seg,
                                                    float4* __restrict__ pl_bias, int32_t* __restrict__ pl_len,
                                                    int32_t* __restrict__ pl_nseg, int64_t* __restrict__ counters) {
    __shared__ int wcnt[8], wpad[8];
    const int a = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const size_t hb = (size_t)bh * NQ, sa = hb + a;
    const int na = slot_items[sa];
    const int pb = partner ? partner[sa] : -1;
    const bool lead = na >= 2 || (na == 1 && (pb < 0 || pb > a));
    if (!lead) {
        if (t == 0) {
            pl_len[sa] = 0;
            pl_nseg[sa] = 0;
        }
        return;
    }
    const int ga = pack_guest ? pack_guest[sa] : -1;
    const bool cross = na == 1 && pb > a;
    const int gb = cross && pack_guest ? pack_guest[hb + pb] : -1;
    const int rows[4] = {a, ga, cross ? pb : a, cross ? gb : ga};
    const uint8_t* mk[4];
    const float* wk[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        mk[q] = rows[q] >= 0 ? mask + (hb + rows[q]) * NK : nullptr;
        wk[q] = (bweight && rows[q] >= 0) ? bweight + (hb + rows[q]) * NK : nullptr;
    }
    const int32_t* ko = k_off + (size_t)bh * (NK + 1);
    const int32_t* po = poff + (size_t)bh * (NK + 1);
    const int per = (NK + 255) / 256, m0 = t * per;
    auto kept = [&](int q, int m) { return mk[q] != nullptr && mk[q][m] != 0; };
    int cnt = 0, pad = 0;
    for (int m = m0; m < m0 + per && m < NK; ++m) {
        if (kept(0, m) || kept(1, m) || kept(2, m) || kept(3, m)) {
            ++cnt;
            pad += (ko[m + 1] - ko[m] + 7) & ~7;
        }
    }
    int ic = cnt, ip = pad;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int yc = __shfl_up_sync(0xffffffffu, ic, o), yp = __shfl_up_sync(0xffffffffu, ip, o);
        if (lane >= o) {
            ic += yc;
            ip += yp;
        }
    }
    if (lane == 31) {
        wcnt[w] = ic;
        wpad[w] = ip;
    }
    __syncthreads();
    int ec = ic - cnt, ep = ip - pad, tot_c = 0, tot_p = 0;
    for (int q = 0; q < 8; ++q) {
        if (q < w) {
            ec += wcnt[q];
            ep += wpad[q];
        }
        tot_c += wcnt[q];
        tot_p += wpad[q];
    }
    const float NI = __int_as_float(0xff800000);
    for (int m = m0; m < m0 + per && m < NK; ++m) {
        const bool k0 = kept(0, m), k1 = kept(1, m), k2 = kept(2, m), k3 = kept(3, m);
        if (!(k0 || k1 || k2 || k3)) continue;
        const int sz = ko[m + 1] - ko[m];
        const size_t e = sa * NK + ec;
        pl_pre[e] = ep;
        pl_seg[e] = make_int2(bh * Npad + po[m], sz);
        auto term = [&](int q, bool k) { return k ? (wk[q] ? (float)log2((double)wk[q][m]) : 0.f) : NI; };
        pl_bias[e] = make_float4(term(0, k0), term(1, k1), term(2, k2), term(3, k3));
        ++ec;
        ep += (sz + 7) & ~7;
    }
    if (t == 0) {
        pl_len[sa] = tot_p;
        pl_nseg[sa] = tot_c;
        const int tiles_q = na >= 2 ? na : (cross ? 2 : 1);
        atomicAdd((unsigned long long*)(counters + PARK_CNT_KEY_TILES),
                  (unsigned long long)tiles_q * (unsigned long long)((tot_p + 127) / 128));
    }
}

// Pairs in lead-cluster order (head by head, clusters in order): one CTA scans
// the per-cluster pair counts.  A cluster with n >= 2 tiles pairs tiles (0, 1),
// (2, 3), ...; a single-tile lead pairs with its partner, or runs alone.
__global__ __launch_bounds__(1024) void k_pairs_emit(int BH, int NQ, const int32_t* __restrict__ slot_items,
                                                     const int32_t* __restrict__ slot_base,
                                                     const int32_t* __restrict__ partner,
                                                     PairItem* __restrict__ pairs, int32_t* __restrict__ pair_count) {
    __shared__ int wsum[32];
    __shared__ int s_base;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const long long nslot = (long long)BH * NQ;
    if (t == 0) s_base = 0;
    __syncthreads();
    for (long long s0 = 0; s0 < nslot; s0 += 1024) {
        const long long slot = s0 + t;
        int cnt = 0, na = 0, pb = -1, a = 0;
        if (slot < nslot) {
            const int bh = (int)(slot / NQ);
            a = (int)(slot - (long long)bh * NQ);
            na = slot_items[slot];
            pb = partner ? partner[slot] : -1;
            cnt = na >= 2 ? (na + 1) / 2 : ((na == 1 && (pb < 0 || pb > a)) ? 1 : 0);
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[w] = incl;
        __syncthreads();
        int woff = 0, tot = 0;
        for (int q = 0; q < 32; ++q) {
            if (q < w) woff += wsum[q];
            tot += wsum[q];
        }
        const int base = s_base + woff + incl - cnt;
        if (cnt > 0) {
            const int sb = slot_base[slot];
            if (na >= 2) {
                for (int q = 0; q < cnt; ++q)
                    pairs[base + q] = PairItem{sb + 2 * q, 2 * q + 1 < na ? sb + 2 * q + 1 : -1, (int)slot};
            } else {
                const long long hb = slot - a;
                pairs[base] = PairItem{sb, pb > a ? slot_base[hb + pb] : -1, (int)slot};
            }
        }
        __syncthreads();
        if (t == 0) s_base += tot;
        __syncthreads();
    }
    if (t == 0) *pair_count = s_base;
}

int launch_pair_schedule(int BH, int NQ, int NK, int Npad, const uint8_t* mask, const int32_t* k_off,
                         const float* bweight, const int32_t* poff, const int32_t* pack_guest,
                         const int32_t* slot_items, const int32_t* slot_base, const int32_t* kv_len, int pairing,
                         int2* cand, int32_t* partner, int32_t* pl_pre, int2* pl_seg, float4* pl_bias,
                         int32_t* pl_len, int32_t* pl_nseg, PairItem* pairs, int32_t* pair_count, int64_t* counters,
                         cudaStream_t st) {
    if (NK > 4096) return PARK_ERR_UNSUPPORTED;
    if (pairing) {
        const size_t sm = (size_t)NK * 5;
        ::park::prof_begin(st);
        k_pair_cand<<<dim3(NQ, BH), 256, sm, st>>>(NQ, NK, mask, k_off, pack_guest, slot_items, kv_len, cand,
                                                   partner);
        PARK_TRY_LAUNCH("k_pair_cand", st);
        const size_t sm2 = (size_t)NQ * kPairKeep * 8 + (size_t)NQ * 8;
        if (sm2 > 48 * 1024 &&
            cudaFuncSetAttribute(k_pair_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2) != cudaSuccess) {
            cudaGetLastError();
            return PARK_ERR_CUDA;
        }
        ::park::prof_begin(st);
        k_pair_select<<<BH, 256, sm2, st>>>(NQ, slot_items, cand, partner);
        PARK_TRY_LAUNCH("k_pair_select", st);
    }
    ::park::prof_begin(st);
    k_pair_lists<<<dim3(NQ, BH), 256, 0, st>>>(NQ, NK, Npad, k_off, mask, bweight, poff, pack_guest, slot_items,
                                               pairing ? partner : nullptr, pl_pre, pl_seg, pl_bias, pl_len, pl_nseg,
                                               counters);
    PARK_TRY_LAUNCH("k_pair_lists", st);
    ::park::prof_begin(st);
    k_pairs_emit<<<1, 1024, 0, st>>>(BH, NQ, slot_items, slot_base, pairing ? partner : nullptr, pairs, pair_count);
    PARK_TRY_LAUNCH("k_pairs_emit", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(352, 1)
    k_sparse_attn_pair(const __grid_constant__ CUtensorMap tmQ, const uint8_t* __restrict__ Kimg,
                       const uint8_t* __restrict__ Vimg, int N, int NK, const int32_t* __restrict__ q_perm,
                       const int2* __restrict__ pl_seg, const float4* __restrict__ pl_bias,
                       const int32_t* __restrict__ pl_nseg, const int32_t* __restrict__ pl_pre,
                       const int32_t* __restrict__ pl_len, const WorkItem* __restrict__ items,
                       const PairItem* __restrict__ pairs, const int32_t* __restrict__ pair_count,
                       uint16_t* __restrict__ O, float sl2e, int32_t* __restrict__ status, uint64_t wait_ns) {
    extern __shared__ __align__(1024) uint8_t dsmem_raw[];
    __shared__ PrSmem sh;
    // 1024-byte aligned operand area: Q_A | Q_B | K0 K1 | V0 V1 (each 32 KB)
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Qs = base;  // Q_X at Qs + 2 X PR_BLK
    uint8_t* Ks = base + 4 * PR_BLK;
    uint8_t* Vs = Ks + 2 * PR_KST * PR_BLK;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort = &sh.abort;
    if (threadIdx.x == 0) {
        mbar_init(&sh.q_full, 1);
        mbar_init(&sh.q_empty, 1);
        for (int s = 0; s < PR_KST; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], 1);
        }
        for (int s = 0; s < PR_VST; ++s) {
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.v_empty[s], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&sh.s_full[x], 1);
            mbar_init(&sh.p_full[x], 128);
            mbar_init(&sh.pv_done[x], 1);
            mbar_init(&sh.o_empty[x], 128);
        }
        mbar_init(&sh.final_bar, 1);
        sh.abort = 0;
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) tma_prefetch_desc(&tmQ);
    if (warp == 1) {
        tmem_alloc(&sh.tmem_base, PR_TMEM_COLS);
        tmem_relinquish();
    }
    // K/V stages start as zeros: groups that are never loaded must hold finite values
    for (int i = threadIdx.x; i < 2 * (PR_KST + PR_VST) * PR_BLK / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(Ks)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int n_pairs = *pair_count;
    const uint32_t idS = idesc_bf16(128, 128, 0, 0);   // S = Q K^T: both K-major
    const uint32_t idPV = idesc_bf16(128, 128, 0, 1);  // O += P V: P K-major (TMEM), V MN-major

    if (warp == 0 || warp == 10) {
        // ------------------------------------------------------------ producers
        const bool isK = warp == 0;
        int T = 0, I = 0;
        int k_last[PR_KST], v_last[PR_VST];
        for (int q = 0; q < PR_KST; ++q) k_last[q] = -1;
        for (int q = 0; q < PR_VST; ++q) v_last[q] = -1;
        int q_pending = 0, q_parity = 0;
        for (int it = blockIdx.x; it < n_pairs && !pr_warp_abort(abort); it += gridDim.x) {
            const PairItem pi = pairs[it];
            const int L = pl_len[pi.lead];
            const int nkt = (L + PR_ROWS - 1) / PR_ROWS;
            if (nkt == 0) continue;
            const int nk = pl_nseg[pi.lead];
            const int32_t* pre = pl_pre + (size_t)pi.lead * NK;
            const int2* segs_item = pl_seg + (size_t)pi.lead * NK;
            const float4* bias_item = pl_bias + (size_t)pi.lead * NK;
            if (isK && lane == 0) {
                bool ok = I == 0 || mbar_wait(&sh.q_empty, (I - 1) & 1, abort, wait_ns);
                if (ok) {
                    const int two = pi.ib >= 0;
                    mbar_arrive_expect_tx(&sh.q_full, (two ? 4 : 2) * PR_BLK);
                    tma_load_2d(Qs, &tmQ, &sh.q_full, 0, pi.ia * PR_ROWS);
                    tma_load_2d(Qs + PR_BLK, &tmQ, &sh.q_full, 64, pi.ia * PR_ROWS);
                    if (two) {
                        tma_load_2d(Qs + 2 * PR_BLK, &tmQ, &sh.q_full, 0, pi.ib * PR_ROWS);
                        tma_load_2d(Qs + 3 * PR_BLK, &tmQ, &sh.q_full, 64, pi.ib * PR_ROWS);
                    }
                    q_pending = 1;
                    q_parity = I & 1;
                }
            }
            __syncwarp();
            if (pr_warp_abort(abort)) break;
            // Segment cursor: lane l holds entry seg0 + l of the pair's kept segments
            // (prefix of padded sizes, first padded row, size, logit terms); a tile
            // spans at most 17 segments (each is >= 8 rows), so 32 lanes cover it.
            int seg0 = 0, p_l = 0x7fffffff, src_l = 0, sz_l = 0;
            float4 lw_l = make_float4(0.f, 0.f, 0.f, 0.f);
            auto load_entries = [&](int s0) {
                const int idx = s0 + lane;
                if (idx < nk) {
                    p_l = pre[idx];
                    const int2 e = segs_item[idx];
                    src_l = e.x;
                    sz_l = e.y;
                    lw_l = bias_item[idx];
                } else {
                    p_l = 0x7fffffff;
                    src_l = 0;
                    sz_l = 0;
                    lw_l = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            };
            load_entries(0);
            bool ok = true;
            for (int j = 0; j < nkt && ok; ++j) {
                const int stg = T % PR_VST, round = T / PR_VST;
                int nvalid = 0;                                      // real key rows of group `lane` (V warp)
                float4 lwv = make_float4(0.f, 0.f, 0.f, 0.f);       // and the logit terms of its segment
#pragma unroll 4
                for (int g = 0; g < 16 && !isK; ++g) {
                    const int vg = j * PR_ROWS + 8 * g;
                    const unsigned bal = __ballot_sync(0xffffffffu, p_l <= vg);
                    const int idx = (__popc(bal) - 1) & 31;
                    const int pp = __shfl_sync(0xffffffffu, p_l, idx);
                    const int sz = __shfl_sync(0xffffffffu, sz_l, idx);
                    const float l0 = __shfl_sync(0xffffffffu, lw_l.x, idx);
                    const float l1 = __shfl_sync(0xffffffffu, lw_l.y, idx);
                    const float l2 = __shfl_sync(0xffffffffu, lw_l.z, idx);
                    const float l3 = __shfl_sync(0xffffffffu, lw_l.w, idx);
                    if (lane == g && vg < L) {
                        const int nv = sz - (vg - pp);
                        nvalid = nv < 0 ? 0 : (nv > 8 ? 8 : nv);
                        lwv = make_float4(l0, l1, l2, l3);
                    }
                }
                // this lane's segment (seg0 + lane) as one piece of whole 8-row groups of the tile
                const int t0 = j * PR_ROWS, t1 = min(t0 + PR_ROWS, L);
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
                    const int vn = (j + 1) * PR_ROWS;
                    if (vn < L) {
                        const unsigned bal = __ballot_sync(0xffffffffu, p_l <= vn);
                        seg0 += __popc(bal) - 1;
                        load_entries(seg0);
                    }
                }
                if (isK) {
                    const int ks = T % PR_KST, kround = T / PR_KST;
                    bool w = true;
                    if (lane == 0 && kround > 0) w = mbar_wait(&sh.k_empty[ks], (kround - 1) & 1, abort, wait_ns);
                    if (__shfl_sync(0xffffffffu, w ? 1 : 0, 0) == 0 || pr_warp_abort(abort)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) mbar_arrive_expect_tx(&sh.k_full[ks], tile_bytes);
                    __syncwarp();
                    if (pc_groups > 0)
                        bulk_load(Ks + ks * 2 * PR_BLK + (pc_start >> 3) * 2048, Kimg + src_off, bytes,
                                  &sh.k_full[ks]);
                    k_last[ks] = kround & 1;
                } else {
                    bool w = true;
                    if (lane == 0 && round > 0) w = mbar_wait(&sh.v_empty[stg], (round - 1) & 1, abort, wait_ns);
                    if (__shfl_sync(0xffffffffu, w ? 1 : 0, 0) == 0 || pr_warp_abort(abort)) {
                        ok = false;
                        break;
                    }
                    if (lane < 16) {
                        const float NI = __int_as_float(0xff800000);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const float lv = v == 0 ? lwv.x : (v == 1 ? lwv.y : (v == 2 ? lwv.z : lwv.w));
                            float4* bp = reinterpret_cast<float4*>(&sh.bias[stg][v][8 * lane]);
                            bp[0] = make_float4(nvalid > 0 ? lv : NI, nvalid > 1 ? lv : NI, nvalid > 2 ? lv : NI,
                                                nvalid > 3 ? lv : NI);
                            bp[1] = make_float4(nvalid > 4 ? lv : NI, nvalid > 5 ? lv : NI, nvalid > 6 ? lv : NI,
                                                nvalid > 7 ? lv : NI);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive_expect_tx(&sh.v_full[stg], tile_bytes);
                    __syncwarp();
                    if (pc_groups > 0)
                        bulk_load(Vs + stg * 2 * PR_BLK + (pc_start >> 3) * 2048, Vimg + src_off, bytes,
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
            for (int s = 0; s < PR_KST; ++s)
                if (k_last[s] >= 0) mbar_wait(&sh.k_full[s], k_last[s], &dummy, 100000000ull);
            for (int s = 0; s < PR_VST; ++s)
                if (v_last[s] >= 0) mbar_wait(&sh.v_full[s], v_last[s], &dummy, 100000000ull);
            if (q_pending) mbar_wait(&sh.q_full, q_parity, &dummy, 100000000ull);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int G = 0, I = 0;
            int tc[2] = {0, 0};   // tiles issued per group (phases of p_full, s_full, pv_done)
            int ic[2] = {0, 0};   // items finished per group (phases of o_empty)
            bool ok = true;
            auto issue_S = [&](int x, int g) {
                const uint32_t qa = smem_u32(Qs + 2 * x * PR_BLK);
                const uint32_t ka = smem_u32(Ks + (g % PR_KST) * 2 * PR_BLK);
                const uint32_t d = tmem + (uint32_t)(x * 128);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t qoff = (uint32_t)((kk >> 2) * PR_BLK + (kk & 3) * 32);
                    const uint32_t koff = (uint32_t)((kk >> 2) * 1024 + (kk & 3) * 32);
                    umma_bf16(d, sdesc_sw128(qa + qoff, 16, 1024), sdesc_sw128(ka + koff, 16, 2048), idS, kk > 0);
                }
                umma_commit(&sh.s_full[x]);
            };
            auto issue_PV = [&](int x, int g, int j) {
                const uint32_t va = smem_u32(Vs + (g % PR_VST) * 2 * PR_BLK);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16_ts(tmem + 256u + (uint32_t)(x * 128), tmem + (uint32_t)(x * 128 + 8 * kk),
                                 sdesc_sw128(va + (uint32_t)kk * 4096, 1024, 2048), idPV, (j > 0 || kk > 0));
                umma_commit(&sh.pv_done[x]);
            };
            for (int it = blockIdx.x; it < n_pairs && ok && !*abort; it += gridDim.x) {
                const PairItem pi = pairs[it];
                const int L = pl_len[pi.lead];
                const int nkt = (L + PR_ROWS - 1) / PR_ROWS;
                if (nkt == 0) continue;
                const int nx = pi.ib >= 0 ? 2 : 1;
                if (!mbar_wait(&sh.q_full, I & 1, abort, wait_ns) ||
                    !mbar_wait(&sh.k_full[G % PR_KST], (G / PR_KST) & 1, abort, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int x = 0; x < nx; ++x) issue_S(x, G);
                umma_commit(&sh.k_empty[G % PR_KST]);
                for (int j = 0; j < nkt && ok; ++j) {
                    const int g = G + j;
                    if (!mbar_wait(&sh.v_full[g % PR_VST], (g / PR_VST) & 1, abort, wait_ns)) {
                        ok = false;
                        break;
                    }
                    const bool next = j + 1 < nkt;
                    if (next && !mbar_wait(&sh.k_full[(g + 1) % PR_KST], ((g + 1) / PR_KST) & 1, abort, wait_ns)) {
                        ok = false;
                        break;
                    }
                    for (int x = 0; x < nx; ++x) {
                        // P_X(j) written; O_X read by the epilogue of this group's previous item
                        if (!mbar_wait(&sh.p_full[x], tc[x] & 1, abort, wait_ns) ||
                            (j == 0 && ic[x] > 0 && !mbar_wait(&sh.o_empty[x], (ic[x] - 1) & 1, abort, wait_ns))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_PV(x, g, j);
                        ++tc[x];
                        if (next) issue_S(x, g + 1);
                    }
                    if (!ok) break;
                    umma_commit(&sh.v_empty[g % PR_VST]);
                    if (next) umma_commit(&sh.k_empty[(g + 1) % PR_KST]);
                }
                if (!ok) break;
                umma_commit(&sh.q_empty);
                for (int x = 0; x < nx; ++x) ++ic[x];
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
        const int x = (warp - 2) >> 2;   // 0: first tile of the pair (warps 2-5), 1: second (6-9)
        const int quad = warp & 3;       // TMEM lane quadrant of this warp
        const int row = 32 * quad + lane;
        const uint32_t trow = tmem + ((uint32_t)(32 * quad) << 16);
        const uint32_t sX = (uint32_t)(x * 128), oX = 256u + (uint32_t)(x * 128);
        const float2 sl2e2 = make_float2(sl2e, sl2e);
        const float NEG = __int_as_float(0xff800000);
        int G = 0, tX = 0;
        // Waits are decided per warp; after a failed wait the warp skips every later
        // wait and all tensor-memory work but still walks the items.
        bool failed = false;
        auto wwait = [&](uint64_t* bar, uint32_t parity) {
            if (!failed) failed = !__all_sync(0xffffffffu, mbar_wait(bar, parity, abort, wait_ns));
            return !failed;
        };
        for (int it = blockIdx.x; it < n_pairs; it += gridDim.x) {
            const PairItem pi = pairs[it];
            const int L = pl_len[pi.lead];
            const int nkt = (L + PR_ROWS - 1) / PR_ROWS;
            if (nkt == 0) continue;
            const int my = x == 0 ? pi.ia : pi.ib;
            if (my < 0) {  // a single: the second group idles
                G += nkt;
                continue;
            }
            const WorkItem wi = items[my];
            const int grp = 2 * x + (row < wi.rows ? 0 : 1);  // own or guest rows
            float m_ref = NEG;
            float2 l2 = make_float2(0.f, 0.f);
            for (int j = 0; j < nkt; ++j, ++tX) {
                const int g = G + j, vs = g % PR_VST;
                const bool live = wwait(&sh.s_full[x], tX & 1) && wwait(&sh.v_full[vs], (g / PR_VST) & 1);
                if (!live) continue;
                tc_fence_after();
                // pass 1: logits with their column bias, written back in place; row maximum
                const float* bz = sh.bias[vs][grp];
                float tm0 = NEG, tm1 = NEG;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t s[32];
                    tmem_ld32(trow + sX + (uint32_t)(32 * c), s);
                    tmem_ld_wait();
                    tmem_ld_dep(s);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 bb = *reinterpret_cast<const float4*>(bz + 32 * c + 4 * q);
                        const float2 x01 = __ffma2_rn(make_float2(pr_bits(s[4 * q]), pr_bits(s[4 * q + 1])), sl2e2,
                                                      make_float2(bb.x, bb.y));
                        const float2 x23 = __ffma2_rn(make_float2(pr_bits(s[4 * q + 2]), pr_bits(s[4 * q + 3])),
                                                      sl2e2, make_float2(bb.z, bb.w));
                        s[4 * q + 0] = __float_as_uint(x01.x);
                        s[4 * q + 1] = __float_as_uint(x01.y);
                        s[4 * q + 2] = __float_as_uint(x23.x);
                        s[4 * q + 3] = __float_as_uint(x23.y);
                        tm0 = pr_max3(tm0, x01.x, x01.y);
                        tm1 = pr_max3(tm1, x23.x, x23.y);
                    }
                    tmem_st32(trow + sX + (uint32_t)(32 * c), s);
                }
                tmem_st_wait();
                const float tmax = fmaxf(tm0, tm1);
                if (j == 0) {
                    m_ref = tmax;
                } else if (__any_sync(0xffffffffu, tmax > m_ref + kRescaleThr)) {
                    // decided per warp; rows that keep their reference get alpha = 1.  O must
                    // hold PV_{j-1}.
                    if (!wwait(&sh.pv_done[x], (tX - 1) & 1)) continue;
                    tc_fence_after();
                    const float m_new = tmax > m_ref + kRescaleThr ? tmax : m_ref;
                    const float alpha = pr_ex2(m_ref - m_new);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tmem_ld32(trow + oX + (uint32_t)(32 * c), o);
                        tmem_ld_wait();
                        tmem_ld_dep(o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(pr_bits(o[e]) * alpha);
                        tmem_st32(trow + oX + (uint32_t)(32 * c), o);
                    }
                    tmem_st_wait();
                    l2.x *= alpha;
                    l2.y *= alpha;
                    m_ref = m_new;
                }
                // pass 2: P = 2^(logit - reference) as bf16 pairs over the first 64 columns.
                // A row that has met only masked keys so far (a guest row can) keeps
                // m_ref = -inf: its P is 0, and the first real maximum rescales O by 0.
                const float mr = m_ref == NEG ? 0.f : m_ref;
                const float2 nm2 = make_float2(-mr, -mr);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t s[32];
                    tmem_ld32(trow + sX + (uint32_t)(32 * c), s);
                    tmem_ld_wait();
                    tmem_ld_dep(s);
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 d = __fadd2_rn(make_float2(pr_bits(s[2 * e]), pr_bits(s[2 * e + 1])), nm2);
                        const float p0 = pr_ex2(d.x), p1 = pr_ex2(d.y);
                        l2 = __fadd2_rn(l2, make_float2(p0, p1));
                        __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                        pk[e] = *reinterpret_cast<uint32_t*>(&h);
                    }
                    tmem_st16(trow + sX + (uint32_t)(16 * c), pk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&sh.p_full[x]);
            }
            G += nkt;
            // epilogue: O / l, original token order
            if (!wwait(&sh.pv_done[x], (tX - 1) & 1)) continue;
            tc_fence_after();
            const float lt = l2.x + l2.y;
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            const int grow = row - wi.rows;  // row of the guest part, if any
            const bool has = row < wi.rows || grow < wi.g_rows;
            const int tok = !has ? 0
                                 : (row < wi.rows ? q_perm[(size_t)wi.bh * N + wi.q_start + row]
                                                  : q_perm[(size_t)wi.bh * N + wi.g_start + grow]);
            uint4* dst = reinterpret_cast<uint4*>(O + ((size_t)wi.bh * N + tok) * 128);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(trow + oX + (uint32_t)(32 * c), o);
                tmem_ld_wait();
                tmem_ld_dep(o);
                if (has) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 h = __floats2bfloat162_rn(pr_bits(o[8 * q + 2 * e]) * inv,
                                                                     pr_bits(o[8 * q + 2 * e + 1]) * inv);
                            w4[e] = *reinterpret_cast<uint32_t*>(&h);
                        }
                        dst[4 * c + q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&sh.o_empty[x]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, PR_TMEM_COLS);
    }
    if (threadIdx.x == 0 && sh.abort) set_status(status, PARK_ERR_TIMEOUT);
}

size_t attn_pair_smem_bytes() { return (size_t)(4 + 2 * PR_KST + 2 * PR_VST) * PR_BLK + 1024; }

int launch_sparse_attn_pair(const void* Qimg, size_t item_cap, const void* Kpad, const void* Vpad, int N, int NK,
                            const int32_t* q_perm, const int2* pl_seg, const float4* pl_bias, const int32_t* pl_nseg,
                            const int32_t* pl_pre, const int32_t* pl_len, const WorkItem* items, const PairItem* pairs,
                            const int32_t* pair_count, void* O, int32_t* status, int num_sms, cudaStream_t st) {
    CUtensorMap mQ;
    PARK_CHECK(make_tma_map_bf16(&mQ, Qimg, (uint64_t)item_cap * PR_ROWS, 128, 128));
    const size_t sm = attn_pair_smem_bytes();
    cudaFuncSetAttribute(k_sparse_attn_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    const float sl2e = (1.0f / sqrtf(128.f)) * kLog2e;
    ::park::prof_begin(st);
    k_sparse_attn_pair<<<num_sms, 352, sm, st>>>(mQ, (const uint8_t*)Kpad, (const uint8_t*)Vpad, N, NK, q_perm, pl_seg,
                                                 pl_bias, pl_nseg, pl_pre, pl_len, items, pairs, pair_count,
                                                 (uint16_t*)O, sl2e, status, wait_limit_ns());
    PARK_TRY_LAUNCH("k_sparse_attn_pair", st);
    return PARK_OK;
}

}  // namespace park
