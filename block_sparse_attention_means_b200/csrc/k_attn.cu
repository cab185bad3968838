// Block-sparse attention over the kept (query cluster, key cluster) pairs
// (PARK abstract: attention is computed inside the retrieved blocks alone).
//
// Layout: Q, K, V are first gathered into cluster-contiguous order (q_perm /
// k_perm), so every query cluster is a run of rows and every key cluster a run
// of rows.  The schedule turns each non-empty query cluster into 64-row query
// tiles and, for the cluster's kept key clusters (CSR, ascending m), a prefix
// of their sizes: the kept keys form one virtual sequence that is cut into full
// 64-row key tiles, so key clusters smaller than a tile share a tile (the
// gather-into-full-tiles idea of the AB-Attention article).  A persistent
// kernel takes query tiles from a work counter; each tile runs an online
// Softmax over its virtual key tiles and writes O rows back in original token
// order.
#include "kernels.h"

namespace park {

// ---------------------------------------------------------------- gather
__global__ void k_gather_rows(const uint4* __restrict__ X, const int32_t* __restrict__ perm, uint4* __restrict__ Xp,
                              size_t rows, int N, int vpr) {
    size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < rows * vpr; e += stride) {
        size_t row = e / vpr;
        int pc = (int)(e - row * vpr);
        size_t bh = row / N;
        size_t src = bh * N + perm[row];
        Xp[e] = X[src * vpr + pc];
    }
}

int launch_gather(const void* X, int dtype, int BH, int N, int D, const int32_t* perm, void* Xp, cudaStream_t st) {
    int vpr = D * (dtype == PARK_BF16 ? 2 : 4) / 16;
    size_t rows = (size_t)BH * N;
    size_t total = rows * vpr;
    int blocks = (int)((total + 255) / 256);
    ::park::prof_begin(st);
    if (blocks > 148 * 32) blocks = 148 * 32;
    k_gather_rows<<<blocks, 256, 0, st>>>((const uint4*)X, perm, (uint4*)Xp, rows, N, vpr);
    PARK_TRY_LAUNCH("k_gather_rows", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- schedule
// One CTA per (query cluster, head): kv_pre[j] = sum of the sizes of the first
// j kept key clusters (rounded up to multiples of 8 when pad8 is set); kv_len =
// their total; query tiles appended to the work list.  Counters: attended
// query-key pairs (unpadded) and work items.
__global__ __launch_bounds__(256) void k_attn_schedule(int NQ, int NK, const int32_t* __restrict__ q_off,
                                                       const int32_t* __restrict__ k_off,
                                                       const int32_t* __restrict__ kept_ptr,
                                                       const int32_t* __restrict__ kept_idx,
                                                       int32_t* __restrict__ kv_pre, int32_t* __restrict__ kv_len,
                                                       WorkItem* __restrict__ items, int32_t* __restrict__ item_count,
                                                       int64_t* __restrict__ counters, int tile_rows, int pad8,
                                                       const int32_t* __restrict__ poff, int Npad,
                                                       int2* __restrict__ segs, const float* __restrict__ bweight,
                                                       float* __restrict__ segw) {
    __shared__ int wsum[8], wsum_u[8];
    const int r = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int qs = q_off[(size_t)bh * (NQ + 1) + r], nr = q_off[(size_t)bh * (NQ + 1) + r + 1] - qs;
    const int kp0 = kept_ptr[(size_t)bh * (NQ + 1) + r], nk = kept_ptr[(size_t)bh * (NQ + 1) + r + 1] - kp0;
    const int32_t* kl = kept_idx + (size_t)bh * NQ * NK + kp0;
    int32_t* pre = kv_pre + (size_t)bh * NQ * NK + kp0;
    const int32_t* ko = k_off + (size_t)bh * (NK + 1);
    auto padded = [&](int sz) { return pad8 ? (sz + 7) & ~7 : sz; };
    const int seg = (nk + 255) / 256, b0 = t * seg;
    int loc = 0, loc_u = 0;
    for (int e = b0; e < b0 + seg && e < nk; ++e) {
        const int sz = ko[kl[e] + 1] - ko[kl[e]];
        loc += padded(sz);
        loc_u += sz;
    }
    int incl = loc, su = loc_u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
        su += __shfl_xor_sync(0xffffffffu, su, o);
    }
    if (lane == 31) wsum[w] = incl;
    if (lane == 0) wsum_u[w] = su;
    __syncthreads();
    int woff = 0, total = 0, total_u = 0;
    for (int q = 0; q < 8; ++q) {
        if (q < w) woff += wsum[q];
        total += wsum[q];
        total_u += wsum_u[q];
    }
    int run = woff + incl - loc;
    for (int e = b0; e < b0 + seg && e < nk; ++e) {
        const int m = kl[e], sz = ko[m + 1] - ko[m];
        pre[e] = run;
        if (segs) segs[(size_t)bh * NQ * NK + kp0 + e] = make_int2(bh * Npad + poff[(size_t)bh * (NK + 1) + m], sz);
        // additive logit term of the segment (log2 of its SIP weight; 0 without weights)
        if (segw) segw[(size_t)bh * NQ * NK + kp0 + e] =
                      bweight ? (float)log2((double)bweight[((size_t)bh * NQ + r) * NK + m]) : 0.f;
        run += padded(sz);
    }
    if (t == 0) {
        kv_len[(size_t)bh * NQ + r] = nr > 0 ? total : 0;
        if (nr > 0 && total > 0) {
            int tiles = (nr + tile_rows - 1) / tile_rows;
            int base = atomicAdd(item_count, tiles);
            for (int q = 0; q < tiles; ++q) {
                WorkItem it;
                it.bh = bh;
                it.r = r;
                it.q_start = qs + q * tile_rows;
                it.rows = min(tile_rows, nr - q * tile_rows);
                it.g = -1;
                it.g_start = 0;
                it.g_rows = 0;
                items[base + q] = it;
            }
            atomicAdd((unsigned long long*)(counters + PARK_CNT_KEPT_PAIRS),
                      (unsigned long long)nr * (unsigned long long)total_u);
            atomicAdd((unsigned long long*)(counters + PARK_CNT_WORK_ITEMS), (unsigned long long)tiles);
            // (query tile, key tile) products: 128 x 128 on the tensor-core path, whose
            // items are up to two 128-row query halves
            const int qt = pad8 ? (nr + 127) / 128 : tiles, kt = pad8 ? (total + 127) / 128 : (total + tile_rows - 1) / tile_rows;
            atomicAdd((unsigned long long*)(counters + PARK_CNT_KEY_TILES),
                      (unsigned long long)qt * (unsigned long long)kt);
        }
    }
}

int launch_attn_schedule(int BH, int NQ, int NK, const int32_t* q_off, const int32_t* k_off,
                         const int32_t* kept_ptr, const int32_t* kept_idx, int32_t* kv_pre, int32_t* kv_len,
                         WorkItem* items, int32_t* item_count, int64_t* counters, int tile_rows, int pad8,
                         const int32_t* poff, int Npad, int2* segs, const float* bweight, float* segw,
                         cudaStream_t st) {
    ::park::prof_begin(st);
    k_attn_schedule<<<dim3(NQ, BH), 256, 0, st>>>(NQ, NK, q_off, k_off, kept_ptr, kept_idx, kv_pre, kv_len, items,
                                                  item_count, counters, tile_rows, pad8, poff, Npad, segs, bweight,
                                                  segw);
    PARK_TRY_LAUNCH("k_attn_schedule", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- query-tile packing
// A guest g (more than one 128-row tile, last tile of rem rows) may join the
// single tile of a host h (1 <= n_h <= 128 - rem): gain = T_g + T_h - T(g u h)
// key tiles, T(L) = ceil(L / 16) for L kept 8-row groups, the shared groups
// counted from the bit planes as in the merge.  k_pack_cand: one CTA per
// (cluster, head) lists a guest's kPackCand best hosts (gain, then lowest h);
// k_pack_select: one warp per head takes the guests in cluster order, each
// joining its best listed host not yet taken (lane k holds the guest's k-th
// listed host; a ballot finds the first one free, before the end of the list).
constexpr int kPackCand = kPackCandidates;

__global__ __launch_bounds__(256) void k_pack_cand(int NQ, int Wd, MergeWs m, int2* __restrict__ cand) {
    extern __shared__ uint32_t pk_sm[];
    uint32_t* sg = pk_sm;                                   // [nb][Wd] guest S & P_b
    int* gain = reinterpret_cast<int*>(pk_sm + kMergePlanes * Wd);  // [NQ]
    const int g = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const size_t hb = (size_t)bh * NQ;
    int2* out = cand + (hb + g) * kPackCand;
    const int ng = m.n[hb + g];
    if (ng <= 128) {  // not a guest
        if (tid < kPackCand) out[tid] = make_int2(0, -1);
        return;
    }
    const int nb = m.nb[bh];
    const int rem = ((ng - 1) & 127) + 1;
    const int Lg = m.L[hb + g], Tg = (Lg + 15) >> 4;
    for (int i = tid; i < nb * Wd; i += blockDim.x) {
        const int b = i / Wd, w = i - b * Wd;
        sg[i] = m.S[(hb + g) * Wd + w] & m.P[((size_t)bh * kMergePlanes + b) * Wd + w];
    }
    __syncthreads();
    for (int h = tid; h < NQ; h += blockDim.x) {
        const int nh = m.n[hb + h];
        int gv = 0;
        if (nh >= 1 && nh <= 128 - rem) {
            const int Lh = m.L[hb + h], Th = (Lh + 15) >> 4;
            int inter = 0;
            const uint32_t* Sh = m.S + (hb + h) * Wd;
            for (int w = 0; w < Wd; ++w) {
                const uint32_t x = Sh[w];
                if (!x) continue;
                for (int b = 0; b < nb; ++b) inter += __popc(x & sg[b * Wd + w]) << b;
            }
            gv = Tg + Th - ((Lg + Lh - inter + 15) >> 4);
        }
        gain[h] = gv;
    }
    __syncthreads();
    if (tid < 32) {  // one warp: the kPackCand largest positive gains, ties to the lowest h
        const int lane = tid;
        for (int k = 0; k < kPackCand; ++k) {
            int bg = 0, bi = -1;
            for (int h = lane; h < NQ; h += 32)
                if (gain[h] > bg) {
                    bg = gain[h];
                    bi = h;
                }
            for (int o = 16; o > 0; o >>= 1) {
                const int go = __shfl_xor_sync(0xffffffffu, bg, o), ho = __shfl_xor_sync(0xffffffffu, bi, o);
                if (go > bg || (go == bg && ho >= 0 && (bi < 0 || ho < bi))) {
                    bg = go;
                    bi = ho;
                }
            }
            if (lane == 0) out[k] = make_int2(bg, bi);
            if (bi >= 0 && lane == (bi & 31)) gain[bi] = 0;  // taken out of the next round
            __syncwarp();
        }
    }
}

__global__ void k_pack_select(int NQ, const MergeWs m, const int2* __restrict__ cand, int32_t* __restrict__ pack_host,
                              int32_t* __restrict__ pack_guest) {
    static_assert(kPackCand == 32, "one listed host per lane");
    extern __shared__ uint32_t taken[];                    // [ceil(NQ / 32)] hosts already taken
    uint8_t* guest = reinterpret_cast<uint8_t*>(taken + (NQ + 31) / 32);  // [NQ] cluster spills over a tile
    const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const size_t hb = (size_t)bh * NQ;
    for (int r = tid; r < NQ; r += blockDim.x) {
        pack_host[hb + r] = -1;
        pack_guest[hb + r] = -1;
        guest[r] = m.n[hb + r] > 128 ? 1 : 0;
    }
    for (int i = tid; i < (NQ + 31) / 32; i += blockDim.x) taken[i] = 0u;
    __syncthreads();
    if (tid >= 32) return;
    int g = 0;
    while (g < NQ && !guest[g]) ++g;
    int2 e = g < NQ ? cand[(hb + g) * kPackCand + lane] : make_int2(0, -1);
    while (g < NQ) {
        // the next guest's list is loaded while this one is decided
        int gn = g + 1;
        while (gn < NQ && !guest[gn]) ++gn;
        const int2 en = gn < NQ ? cand[(hb + gn) * kPackCand + lane] : make_int2(0, -1);
        const unsigned end = __ballot_sync(0xffffffffu, e.y < 0 || e.x <= 0);
        const int first_end = end ? __ffs(end) - 1 : 32;
        const int hy = e.y < 0 ? 0 : e.y;  // (entries past the end of the list are not read as hosts)
        const bool free_host = lane < first_end && !((taken[hy >> 5] >> (hy & 31)) & 1u);
        const unsigned ok = __ballot_sync(0xffffffffu, free_host);
        if (ok) {
            const int h = __shfl_sync(0xffffffffu, e.y, __ffs(ok) - 1);
            if (lane == 0) {
                taken[h >> 5] |= 1u << (h & 31);
                pack_host[hb + g] = h;
                pack_guest[hb + h] = g;
            }
        }
        __syncwarp();
        g = gn;
        e = en;
    }
}

int launch_pack_pairs(int BH, int NQ, int NK, const uint8_t* mask, const int32_t* q_off, const int32_t* k_off,
                      const MergeWs& m, int2* cand, int32_t* pack_host, int32_t* pack_guest, cudaStream_t st) {
    const int Wd = (NK + 31) / 32;
    PARK_CHECK(launch_merge_setup(mask, q_off, k_off, BH, NQ, NK, m, st));
    const size_t sm = (size_t)kMergePlanes * Wd * 4 + (size_t)NQ * 4;
    if (cudaFuncSetAttribute(k_pack_cand, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess) {
        cudaGetLastError();
        return PARK_ERR_CUDA;
    }
    ::park::prof_begin(st);
    k_pack_cand<<<dim3(NQ, BH), 256, sm, st>>>(NQ, Wd, m, cand);
    PARK_TRY_LAUNCH("k_pack_cand", st);
    ::park::prof_begin(st);
    k_pack_select<<<BH, 256, (size_t)((NQ + 31) / 32) * 4 + (size_t)NQ, st>>>(NQ, m, cand, pack_host, pack_guest);
    PARK_TRY_LAUNCH("k_pack_select", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- schedule (tensor cores)
// One CTA per (query cluster, head).  The slot's key list is the cluster's kept
// set, or for a host the union with its guest's; entries in ascending m.
__global__ __launch_bounds__(256) void k_attn_schedule_tc(int NQ, int NK, int Npad, const int32_t* __restrict__ q_off,
                                                          const int32_t* __restrict__ k_off,
                                                          const uint8_t* __restrict__ mask,
                                                          const float* __restrict__ bweight,
                                                          const int32_t* __restrict__ poff,
                                                          const int32_t* __restrict__ pack_host,
                                                          const int32_t* __restrict__ pack_guest,
                                                          int32_t* __restrict__ kv_pre, int32_t* __restrict__ kv_len,
                                                          int32_t* __restrict__ kv_nseg, int2* __restrict__ segs,
                                                          float* __restrict__ segwA, float* __restrict__ segwB,
                                                          int32_t* __restrict__ slot_items,
                                                          int64_t* __restrict__ counters) {
    __shared__ int wcnt[8], wpad[8];
    __shared__ long long wown[8];
    const int r = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const size_t slot = (size_t)bh * NQ + r;
    const int qs = q_off[(size_t)bh * (NQ + 1) + r], nr = q_off[(size_t)bh * (NQ + 1) + r + 1] - qs;
    const int g = pack_guest ? pack_guest[slot] : -1;  // guest hosted in r's tile
    const int h = pack_host ? pack_host[slot] : -1;    // host of r's last tile
    const uint8_t* mA = mask + slot * NK;
    const uint8_t* mB = g >= 0 ? mask + ((size_t)bh * NQ + g) * NK : nullptr;
    const int32_t* ko = k_off + (size_t)bh * (NK + 1);
    const int32_t* po = poff + (size_t)bh * (NK + 1);
    const int per = (NK + 255) / 256, m0 = t * per;
    int cnt = 0, pad = 0;
    long long own = 0;
    for (int m = m0; m < m0 + per && m < NK; ++m) {
        const bool a = mA[m] != 0, b = mB && mB[m] != 0;
        if (a || b) {
            const int sz = ko[m + 1] - ko[m];
            ++cnt;
            pad += (sz + 7) & ~7;
            if (a) own += sz;
        }
    }
    // block exclusive scans of the entry count and the padded rows
    int ic = cnt, ip = pad;
    long long so = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int yc = __shfl_up_sync(0xffffffffu, ic, o), yp = __shfl_up_sync(0xffffffffu, ip, o);
        if (lane >= o) {
            ic += yc;
            ip += yp;
        }
        so += __shfl_xor_sync(0xffffffffu, so, o);
    }
    if (lane == 31) {
        wcnt[w] = ic;
        wpad[w] = ip;
    }
    if (lane == 0) wown[w] = so;
    __syncthreads();
    int ec = ic - cnt, ep = ip - pad, tot_c = 0, tot_p = 0;
    long long tot_own = 0;
    for (int q = 0; q < 8; ++q) {
        if (q < w) {
            ec += wcnt[q];
            ep += wpad[q];
        }
        tot_c += wcnt[q];
        tot_p += wpad[q];
        tot_own += wown[q];
    }
    const float NI = __int_as_float(0xff800000);
    const float* wA = bweight ? bweight + slot * NK : nullptr;
    const float* wB = (bweight && g >= 0) ? bweight + ((size_t)bh * NQ + g) * NK : nullptr;
    for (int m = m0; m < m0 + per && m < NK; ++m) {
        const bool a = mA[m] != 0, b = mB && mB[m] != 0;
        if (!(a || b)) continue;
        const int sz = ko[m + 1] - ko[m];
        const size_t e = slot * NK + ec;
        kv_pre[e] = ep;
        segs[e] = make_int2(bh * Npad + po[m], sz);
        segwA[e] = a ? (wA ? (float)log2((double)wA[m]) : 0.f) : NI;
        segwB[e] = b ? (wB ? (float)log2((double)wB[m]) : 0.f) : NI;
        ++ec;
        ep += (sz + 7) & ~7;
    }
    if (t == 0) {
        kv_len[slot] = nr > 0 ? tot_p : 0;
        kv_nseg[slot] = tot_c;
        slot_items[slot] = 0;
        if (nr > 0 && tot_p > 0) {
            const int tiles = (nr + 127) / 128;
            const int own_items = h >= 0 ? tiles - 1 : tiles;  // a guest's last tile is in its host's item
            slot_items[slot] = own_items;  // k_items_emit writes them, head by head in cluster order
            atomicAdd((unsigned long long*)(counters + PARK_CNT_KEPT_PAIRS),
                      (unsigned long long)nr * (unsigned long long)tot_own);
            atomicAdd((unsigned long long*)(counters + PARK_CNT_WORK_ITEMS), (unsigned long long)own_items);
            atomicAdd((unsigned long long*)(counters + PARK_CNT_KEY_TILES),
                      (unsigned long long)own_items * (unsigned long long)((tot_p + 127) / 128));
        }
    }
}

// Work items in slot order (head by head, clusters in order, so that the
// persistent attention CTAs, which take consecutive items, work on one head's
// key images at a time): one CTA scans the per-slot item counts.
__global__ __launch_bounds__(1024) void k_items_emit(int BH, int NQ, const int32_t* __restrict__ q_off,
                                                     const int32_t* __restrict__ pack_guest,
                                                     const int32_t* __restrict__ slot_items,
                                                     WorkItem* __restrict__ items, int32_t* __restrict__ item_count) {
    __shared__ int wsum[32];
    __shared__ int s_base;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const long long nslot = (long long)BH * NQ;
    if (t == 0) s_base = 0;
    __syncthreads();
    for (long long s0 = 0; s0 < nslot; s0 += 1024) {
        const long long slot = s0 + t;
        const int cnt = slot < nslot ? slot_items[slot] : 0;
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
            const int bh = (int)(slot / NQ), r = (int)(slot - (long long)bh * NQ);
            const int qs = q_off[(size_t)bh * (NQ + 1) + r], nr = q_off[(size_t)bh * (NQ + 1) + r + 1] - qs;
            const int g = pack_guest ? pack_guest[slot] : -1;
            int gs = 0, gr = 0;
            if (g >= 0) {
                const int gq = q_off[(size_t)bh * (NQ + 1) + g], gn = q_off[(size_t)bh * (NQ + 1) + g + 1] - gq;
                gs = gq + 128 * ((gn - 1) / 128);
                gr = gn - 128 * ((gn - 1) / 128);
            }
            for (int q = 0; q < cnt; ++q) {
                WorkItem it;
                it.bh = bh;
                it.r = r;
                it.q_start = qs + q * 128;
                it.rows = min(128, nr - q * 128);
                it.g = g;
                it.g_start = gs;
                it.g_rows = gr;
                items[base + q] = it;
            }
        }
        __syncthreads();
        if (t == 0) s_base += tot;
        __syncthreads();
    }
    if (t == 0) *item_count = s_base;
}

int launch_attn_schedule_tc(int BH, int NQ, int NK, int Npad, const int32_t* q_off, const int32_t* k_off,
                            const uint8_t* mask, const float* bweight, const int32_t* poff, const int32_t* pack_host,
                            const int32_t* pack_guest, int32_t* kv_pre, int32_t* kv_len, int32_t* kv_nseg,
                            int2* segs, float* segwA, float* segwB, int32_t* slot_items, WorkItem* items,
                            int32_t* item_count, int64_t* counters, cudaStream_t st) {
    ::park::prof_begin(st);
    k_attn_schedule_tc<<<dim3(NQ, BH), 256, 0, st>>>(NQ, NK, Npad, q_off, k_off, mask, bweight, poff, pack_host,
                                                     pack_guest, kv_pre, kv_len, kv_nseg, segs, segwA, segwB,
                                                     slot_items, counters);
    PARK_TRY_LAUNCH("k_attn_schedule", st);
    ::park::prof_begin(st);
    k_items_emit<<<1, 1024, 0, st>>>(BH, NQ, q_off, pack_guest, slot_items, items, item_count);
    PARK_TRY_LAUNCH("k_items_emit", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- item-major Q
__global__ void k_item_gather(const uint4* __restrict__ Q, int N, const int32_t* __restrict__ q_perm,
                              const WorkItem* __restrict__ items, const int32_t* __restrict__ item_count,
                              size_t item_cap, uint4* __restrict__ Qimg) {
    constexpr int VPR = 16;  // 16-byte chunks per 128-element bf16 row
    const size_t n = (size_t)min((size_t)*item_count, item_cap) * 128 * VPR;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const size_t rowi = e / VPR;
        const int c = (int)(e - rowi * VPR);
        const size_t it = rowi / 128;
        const int row = (int)(rowi - it * 128);
        const WorkItem wi = items[it];
        const int grow = row - wi.rows;
        int tok = -1;
        if (row < wi.rows) tok = q_perm[(size_t)wi.bh * N + wi.q_start + row];
        else if (grow < wi.g_rows) tok = q_perm[(size_t)wi.bh * N + wi.g_start + grow];
        Qimg[e] = tok >= 0 ? Q[((size_t)wi.bh * N + tok) * VPR + c] : make_uint4(0, 0, 0, 0);
    }
}

int launch_item_gather(const void* Q, int N, const int32_t* q_perm, const WorkItem* items, const int32_t* item_count,
                       size_t item_cap, void* Qimg, int num_sms, cudaStream_t st) {
    ::park::prof_begin(st);
    k_item_gather<<<num_sms * 8, 256, 0, st>>>((const uint4*)Q, N, q_perm, items, item_count, item_cap, (uint4*)Qimg);
    PARK_TRY_LAUNCH("k_item_gather", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- padded K/V
// poff[bh][m] = sum over m' < m of ceil8(|B_m'|) (one CTA per head).
__global__ __launch_bounds__(1024) void k_kv_pad_offsets(const int32_t* __restrict__ k_off, int NK,
                                                         int32_t* __restrict__ poff) {
    __shared__ int wsum[32];
    const int bh = blockIdx.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int32_t* ko = k_off + (size_t)bh * (NK + 1);
    int32_t* po = poff + (size_t)bh * (NK + 1);
    const int seg = (NK + 1023) / 1024, b0 = t * seg;
    int loc = 0;
    for (int m = b0; m < b0 + seg && m < NK; ++m) loc += (ko[m + 1] - ko[m] + 7) & ~7;
    int incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    int woff = 0;
    for (int q = 0; q < w; ++q) woff += wsum[q];
    int run = woff + incl - loc;
    for (int m = b0; m < b0 + seg && m < NK; ++m) {
        po[m] = run;
        run += (ko[m + 1] - ko[m] + 7) & ~7;
    }
    if (b0 < NK && b0 + seg >= NK) po[NK] = run;
}

// Row copies into the padded layout, stored as the byte image of the
// tensor-core kernel's shared-memory tiles: padded row pp of a head lies in
// 8-row group q = pp / 8 (2048 bytes at q * 2048), first the 64-column half 0
// then half 1 (1024 bytes each); inside a half, row r = pp % 8 takes 128 bytes
// at r * 128 and its 16-byte chunk c sits at chunk position c ^ r (the 128-byte
// swizzle).  A run of whole groups is then one contiguous bulk copy.  Pad rows
// are zeros.
__device__ __forceinline__ size_t kv_image_chunk(size_t head_base_groups, int pp, int c) {
    const int q = pp >> 3, r = pp & 7, h = c >> 3, c16 = c & 7;
    return (head_base_groups + (size_t)q) * 128 + (size_t)h * 64 + (size_t)r * 8 + (size_t)(c16 ^ r);
}

__global__ void k_kv_pad_gather(const uint4* __restrict__ K, const uint4* __restrict__ V, int N, int NK, int Npad,
                                size_t BH, const int32_t* __restrict__ k_perm, const int32_t* __restrict__ k_labels,
                                const int32_t* __restrict__ k_off, const int32_t* __restrict__ poff,
                                uint4* __restrict__ Kp, uint4* __restrict__ Vp) {
    constexpr int VPR = 16;  // 16-byte chunks per 128-element bf16 row
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t rows = BH * (size_t)N;
    const size_t gph = (size_t)Npad / 8;  // groups per head
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < rows * VPR; e += stride) {
        const size_t row = e / VPR;
        const int pc = (int)(e - row * VPR);
        const size_t bh = row / N;
        const int pos = (int)(row - bh * N);
        const int tok = k_perm[row];
        const int m = k_labels[bh * N + tok];
        const int pp = poff[bh * (NK + 1) + m] + (pos - k_off[bh * (NK + 1) + m]);
        const size_t dst = kv_image_chunk(bh * gph, pp, pc);
        Kp[dst] = K[(bh * N + tok) * VPR + pc];
        Vp[dst] = V[(bh * N + tok) * VPR + pc];
    }
    // pad rows: at most 7 per cluster
    const size_t pads = BH * (size_t)NK * 7 * VPR;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < pads; e += stride) {
        const size_t q = e / VPR;
        const int pc = (int)(e - q * VPR);
        const size_t bhm = q / 7;
        const int i = (int)(q - bhm * 7);
        const size_t bh = bhm / NK;
        const int m = (int)(bhm - bh * NK);
        const int sz = k_off[bh * (NK + 1) + m + 1] - k_off[bh * (NK + 1) + m];
        const int padn = ((sz + 7) & ~7) - sz;
        if (i < padn) {
            const size_t dst = kv_image_chunk(bh * gph, poff[bh * (NK + 1) + m] + sz + i, pc);
            Kp[dst] = make_uint4(0, 0, 0, 0);
            Vp[dst] = make_uint4(0, 0, 0, 0);
        }
    }
}

int launch_kv_pad_gather(const void* K, const void* V, int BH, int N, int NK, int Npad, const int32_t* k_perm,
                         const int32_t* k_labels, const int32_t* k_off, int32_t* poff, void* Kpad, void* Vpad,
                         cudaStream_t st) {
    ::park::prof_begin(st);
    k_kv_pad_offsets<<<BH, 1024, 0, st>>>(k_off, NK, poff);
    PARK_TRY_LAUNCH("k_kv_pad_offsets", st);
    size_t total = (size_t)BH * N * 16;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    ::park::prof_begin(st);
    k_kv_pad_gather<<<blocks, 256, 0, st>>>((const uint4*)K, (const uint4*)V, N, NK, Npad, (size_t)BH, k_perm,
                                            k_labels, k_off, poff, (uint4*)Kpad, (uint4*)Vpad);
    PARK_TRY_LAUNCH("k_kv_pad_gather", st);
    return PARK_OK;
}

// ---------------------------------------------------------------- attention (float32 inputs)
// One warp per query row: walks the kept key clusters of its query cluster in
// ascending m and their keys in sorted order; online Softmax in float32.
template <typename T>
__global__ void k_sparse_attn_simt(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V, int N,
                                   int D, int NQ, int NK, const int32_t* __restrict__ q_labels,
                                   const int32_t* __restrict__ k_perm, const int32_t* __restrict__ k_off,
                                   const int32_t* __restrict__ kept_ptr, const int32_t* __restrict__ kept_idx,
                                   const float* __restrict__ bweight, T* __restrict__ O, size_t rows, float scale) {
    const int lane = threadIdx.x & 31;
    const size_t nw = ((size_t)gridDim.x * blockDim.x) >> 5;
    for (size_t row = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < rows; row += nw) {
        const size_t bh = row / N;
        const int r = q_labels[row];
        float q[4], o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            int j = lane + 32 * u;
            q[u] = j < D ? Elem<T>::to_float(Q + row * D, j) : 0.f;
            o[u] = 0.f;
        }
        float m = __int_as_float(0xff800000), l = 0.f;
        const int p0 = kept_ptr[bh * (NQ + 1) + r], p1 = kept_ptr[bh * (NQ + 1) + r + 1];
        const int32_t* ko = k_off + bh * (NK + 1);
        for (int e = p0; e < p1; ++e) {
            int mk = kept_idx[bh * NQ * NK + e];
            const float lw = bweight ? logf(bweight[(bh * NQ + r) * NK + mk]) : 0.f;  // SIP weight, natural log
            for (int pos = ko[mk]; pos < ko[mk + 1]; ++pos) {
                size_t tok = bh * N + k_perm[bh * N + pos];
                float sdot = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    int j = lane + 32 * u;
                    if (j < D) sdot = fmaf(q[u], Elem<T>::to_float(K + tok * D, j), sdot);
                }
                float sc = warp_sum(sdot) * scale + lw;
                float mn = fmaxf(m, sc);
                float corr = expf(m - mn), pw = expf(sc - mn);
                l = l * corr + pw;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    int j = lane + 32 * u;
                    float vv = j < D ? Elem<T>::to_float(V + tok * D, j) : 0.f;
                    o[u] = o[u] * corr + pw * vv;
                }
                m = mn;
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            int j = lane + 32 * u;
            if (j < D) {
                const float out = l > 0.f ? o[u] / l : 0.f;
                if (sizeof(T) == 2)
                    reinterpret_cast<uint16_t*>(O)[row * D + j] = __bfloat16_as_ushort(__float2bfloat16_rn(out));
                else
                    reinterpret_cast<float*>(O)[row * D + j] = out;
            }
        }
    }
}

int launch_sparse_attn_simt(const void* Q, const void* K, const void* V, int dtype, int BH, int N, int D, int NQ,
                            int NK, const int32_t* q_labels, const int32_t* k_perm, const int32_t* k_off,
                            const int32_t* kept_ptr, const int32_t* kept_idx, const float* bweight, void* O,
                            cudaStream_t st) {
    if (D > 128) return PARK_ERR_UNSUPPORTED;
    size_t rows = (size_t)BH * N;
    int blocks = (int)((rows * 32 + 255) / 256);
    ::park::prof_begin(st);
    if (blocks > 148 * 64) blocks = 148 * 64;
    if (dtype == PARK_BF16)
        k_sparse_attn_simt<bf16_t><<<blocks, 256, 0, st>>>((const bf16_t*)Q, (const bf16_t*)K, (const bf16_t*)V, N, D,
                                                           NQ, NK, q_labels, k_perm, k_off, kept_ptr, kept_idx, bweight,
                                                           (bf16_t*)O, rows, 1.0f / sqrtf((float)D));
    else
        k_sparse_attn_simt<float><<<blocks, 256, 0, st>>>((const float*)Q, (const float*)K, (const float*)V, N, D, NQ,
                                                          NK, q_labels, k_perm, k_off, kept_ptr, kept_idx, bweight,
                                                          (float*)O, rows, 1.0f / sqrtf((float)D));
    PARK_TRY_LAUNCH("k_sparse_attn_simt", st);
    return PARK_OK;
}

}  // namespace park
