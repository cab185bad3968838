// Internal launch interface between the C ABI (park_api.cu) and the kernels.
// Every launcher enqueues on `st`, never synchronises, and returns a PARK_*
// code (PARK_ERR_CUDA when the launch itself failed).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace park {

// K-means centroid operands for the score GEMM: score_k = bias_k - 2 x . w_k.
struct CentroidOps {
    const uint16_t* w;  // bf16 [BH][K][kw]   (queries: the centroids themselves, kw = D;
                        //                     keys: hi/lo split of M c, kw = 2D)
    int kw;
    float* bias32;      // [BH][bias_ld]  bias rounded to float
    int bias_ld;        // leading dimension of bias32 (multiple of 128, >= K)
    double* bias64;     // [BH][K]  ||c||^2 (queries) or c^T M c (keys)
    double* w64;        // [BH][K][D] M c in float64 (keys only)
    float* wmax;        // [BH] max_k ||w_k||  (rounded up)
    float* bmax;        // [BH] max_k |bias_k| (rounded up)
};

struct Lists {
    int32_t* full_row;  // [BH][N]: per head, bh*N + i of the rows to rescore against every centroid
    int32_t* counts;    // [BH]: rows listed per head (zeroed before each assign)
};

// ---- k_prep.cu
// wide (bf16, may be null): per-head flags, set where an element has
// |x| >= 2^16 (zeroed by the caller); per_head_elems = N * D.  tiny_rows (bf16,
// may be null): one byte per row of row_elems elements, set to 1 where the row
// holds a nonzero element with |x| < 2^-20 (zeroed by the caller).  xnorm (bf16
// with row_elems = 128, may be null): every row's norm, rounded up to float.
int launch_input_check(const void* x, size_t n_elems, int dtype, int32_t* status, int32_t* wide,
                       size_t per_head_elems, uint8_t* tiny_rows, size_t row_elems, float* xnorm,
                       cudaStream_t st);
int launch_metric(const void* Q, int dtype, int BH, int N, int D, double* part, int nchunks, double* M,
                  double* M_out, cudaStream_t st);
int launch_strided_init(const void* X, int dtype, int BH, int N, int D, int K, void* C, cudaStream_t st);
int launch_centroid_prep(const void* C, int dtype, int BH, int K, int D, const double* M, CentroidOps ops,
                         cudaStream_t st);

// ---- k_assign.cu
// k_assign_tc.cu: tcgen05 score GEMM with the certified top-3 epilogue (bf16, D = 128)
int launch_assign_tc(const void* X, int BH, int N, int K, const CentroidOps& ops, const float* xnorm, float gamma,
                     int32_t* labels, Lists lists, int32_t* status, int num_sms, cudaStream_t st);
int launch_recheck(const void* X, int dtype, int BH, int N, int D, int K, const void* C, const double* w64,
                   const double* b64, int32_t* labels, Lists lists, int all_rows, int num_sms,
                   int64_t* counters, int cnt_slot, cudaStream_t st);
// float64 assign of rows row0 .. N-1 of every head against every centroid
int launch_recheck_rows(const void* X, int dtype, int BH, int N, int D, int K, const void* C, const double* w64,
                        const double* b64, int32_t* labels, int row0, int num_sms, cudaStream_t st);

// ---- k_sort.cu
int launch_label_sort(const int32_t* labels, int BH, int N, int K, int32_t* hist, int nchunks, int32_t* perm,
                      int32_t* offsets, cudaStream_t st);
// wide, tiny_rows: the per-head and per-row flags of launch_input_check for X
// (either null: every head takes the general path).
int launch_update(const void* X, int dtype, int BH, int N, int D, int K, const int32_t* perm,
                  const int32_t* offsets, void* C, const int32_t* wide, const uint8_t* tiny_rows,
                  cudaStream_t st);

// ---- k_pama.cu
// size_prior: logits gain log |B_m|.  select: 0 top-p; 1 top-k, the ceil(p L) most
// important (p a ratio); 2 SIP with the uniforms sip_u, writing weight = 1/pi for
// kept blocks and 0 elsewhere.
// k_pama_tc.cu: the importance map and its per-row relative bound rho on tcgen05,
// from Q already gathered into cluster order (Qg [BH][N][128] bf16)
int launch_pama_tc(const void* Qg, int BH, int N, int NQ, int NK, const int32_t* q_perm, const int32_t* q_off,
                   const void* CK, const int32_t* k_off, const float* qnorm, int size_prior, float* importance,
                   float* rho, const float* ckmax, int32_t* status, int num_sms, cudaStream_t st);
size_t pama_tc_smem_bytes(int NK);
int launch_topp(const float* importance, const float* rho, int BH, int NQ, int NK, const int32_t* q_off,
                const int32_t* k_off, float p, int select, const float* sip_u, float* weight, uint8_t* mask,
                int32_t* kept_cnt, float* importance_bound, int32_t* flag_list, int32_t* flag_count,
                cudaStream_t st);
// one row per non-empty query cluster (its centroid), for "w/o PAMA" through launch_pama_f64
int launch_centroid_rows(const int32_t* q_off, int BH, int NQ, int32_t* perm, int32_t* off, cudaStream_t st);
// Float64 PAMA + top-p for the listed clusters (or all): at most kPamaF64Slots
// CTAs, each with pama_f64_scratch_bytes(NK) / kPamaF64Slots bytes of float64
// scratch; work_ctr (zeroed by the caller) hands out the clusters.  one_row:
// every cluster has at most one row (32-row tiles instead of 128).
constexpr int kPamaF64Slots = 160;
size_t pama_f64_scratch_bytes(int NK);
int launch_pama_f64(const void* Q, int dtype, int BH, int N, int D, int NQ, int NK, const int32_t* q_perm,
                    const int32_t* q_off, const void* CK, const int32_t* k_off, float p, int select, int size_prior,
                    const float* sip_u, float* weight, const int32_t* list,
                    const int32_t* count, int all_clusters, int num_sms, int32_t* work_ctr, double* zscratch,
                    float* importance, float* importance_bound, uint8_t* mask, int32_t* kept_cnt, int64_t* counters,
                    cudaStream_t st, int one_row = 0);
int launch_kept_csr(const uint8_t* mask, const int32_t* kept_cnt, int BH, int NQ, int NK, int32_t* kept_ptr,
                    int32_t* kept_idx, int64_t* counters, cudaStream_t st);

// ---- k_hva.cu
// Video-grid windows for the local-window K-means: wt x wh x ww tokens, nWt x
// nWh x nWw of them (nW in all), maxwin tokens in the largest; nvideo = T Hg W.
struct WinGeom {
    int T, Hg, W, wt, wh, ww, nWt, nWh, nWw, nW, nvideo, maxwin;
};
int launch_local_init(const void* X, int dtype, int BH, int N, int D, int K, const WinGeom& g, void* C,
                      cudaStream_t st);
// Grid tokens against their window's centroids; text tokens are left to
// launch_recheck_rows.  C: centroids (Euclidean); w64/b64/wmax/bmax from
// launch_centroid_prep (w64 null: Euclidean).
int launch_assign_local(const void* X, int dtype, int BH, int N, int D, int K, const WinGeom& g, const void* C,
                        const double* w64, const double* b64, const float* wmax, const float* bmax, int32_t* labels,
                        int64_t* counters, int cnt_slot, cudaStream_t st);
size_t local_assign_smem(int K, int nW, int D);
// Rows row0 .. N-1 of every head (the text tokens) against every centroid, with
// the same float32 bound and float64 fallback as launch_assign_local; scratch
// holds text_scratch_bytes(BH, N - row0, K).
size_t text_scratch_bytes(int BH, int n_text, int K);
int launch_assign_text(const void* X, int dtype, int BH, int N, int D, int K, int row0, const void* C,
                       const double* w64, const double* b64, const float* wmax, const float* bmax, void* scratch,
                       int32_t* labels, int64_t* counters, int cnt_slot, cudaStream_t st);
// Query-cluster merging state, per head: S [NQ][Wd] kept-set bitsets, P
// [kMergePlanes][Wd] bit planes of the key clusters' 8-row unit counts, inter
// [NQ][NQ] the kept units two groups share (-1: the pair cannot gain).
constexpr int kMergePlanes = 18;  // unit counts are below 2^18 (N <= 2^20)
constexpr int kMergeMaxNQ = 2048;
struct MergeWs {
    uint32_t* S;
    uint32_t* P;
    int32_t* inter;
    int32_t *n, *L, *alive, *root, *best, *rootf, *todo, *done, *nb;
};
// S, n, L, alive, root, best, P and nb of a MergeWs from the masks (k_merge_init,
// k_merge_planes).
int launch_merge_setup(const uint8_t* mask, const int32_t* q_off, const int32_t* k_off, int BH, int NQ, int NK,
                       const MergeWs& m, cudaStream_t st);
// Rewrites mask rows and kept counts of the merged groups and moves q_labels to
// the groups' roots; `rounds` parallel rounds at most.
int launch_merge(uint8_t* mask, int32_t* kept_cnt, const int32_t* q_off, const int32_t* k_off, int BH, int N, int NQ,
                 int NK, int rounds, const MergeWs& m, int32_t* q_labels, int num_sms, cudaStream_t st);

// ---- k_attn.cu
// One query tile of the attention: rows [q_start, q_start + rows) of cluster r in
// cluster order, and on the tensor-core path optionally the last tile of a guest
// cluster g packed into the same tile (rows [g_start, g_start + g_rows), g = -1
// when none).
struct WorkItem {
    int bh, r, q_start, rows, g, g_start, g_rows;
};
int launch_gather(const void* X, int dtype, int BH, int N, int D, const int32_t* perm, void* Xp, cudaStream_t st);
// pad8: key cluster sizes rounded up to multiples of 8 in kv_pre / kv_len (the
// padded layout of the tensor-core kernel), and segs[j] = (first padded row of
// the j-th kept cluster, its size) written from poff; the pair counter always
// counts the unpadded keys.
int launch_attn_schedule(int BH, int NQ, int NK, const int32_t* q_off, const int32_t* k_off,
                         const int32_t* kept_ptr, const int32_t* kept_idx, int32_t* kv_pre, int32_t* kv_len,
                         WorkItem* items, int32_t* item_count, int64_t* counters, int tile_rows, int pad8,
                         const int32_t* poff, int Npad, int2* segs, const float* bweight, float* segw,
                         cudaStream_t st);
// K and V in key-cluster order with every cluster padded to a multiple of 8
// rows (zeros): poff[bh][m] = first padded row of cluster m; Npad rows per head.
int launch_kv_pad_gather(const void* K, const void* V, int BH, int N, int NK, int Npad, const int32_t* k_perm,
                         const int32_t* k_labels, const int32_t* k_off, int32_t* poff, void* Kpad, void* Vpad,
                         cudaStream_t st);
size_t attn_tc_smem_bytes();
// TMA descriptor for a row-major bf16 [rows][cols] tensor, boxes of 64 columns x
// box_rows, 128-byte swizzle (k_attn_tc.cu).
int make_tma_map_bf16(CUtensorMap* map, const void* ptr, uint64_t rows, uint32_t cols, uint32_t box_rows);
// Query-tile packing for the tensor-core path: the last tile of a query cluster
// with several tiles (a guest) shares the single tile of a cluster with enough
// free rows (its host) when the host tile's key list, the union of both kept
// sets, needs fewer key tiles than the two tiles apart.  Each guest lists its
// best hosts in parallel; then per head, guests in cluster order take the best
// listed host still free.  Uses a MergeWs (S / n / L / P / nb) and cand [BH][NQ][8].
constexpr int kPackCandidates = 32;
int launch_pack_pairs(int BH, int NQ, int NK, const uint8_t* mask, const int32_t* q_off, const int32_t* k_off,
                      const MergeWs& m, int2* cand, int32_t* pack_host, int32_t* pack_guest, cudaStream_t st);
// Tensor-core schedule: per slot (bh, r) the key list at slot * NK (ascending m: padded prefix kv_pre, segs,
// logit terms segwA for the own rows and segwB for the guest rows, -inf where not kept), kv_len, kv_nseg;
// 128-row work items with their guests, head by head in cluster order (slot_items [BH][NQ]
// scratch).  pack_host / pack_guest may be null (no packing).
int launch_attn_schedule_tc(int BH, int NQ, int NK, int Npad, const int32_t* q_off, const int32_t* k_off,
                            const uint8_t* mask, const float* bweight, const int32_t* poff, const int32_t* pack_host,
                            const int32_t* pack_guest, int32_t* kv_pre, int32_t* kv_len, int32_t* kv_nseg,
                            int2* segs, float* segwA, float* segwB, int32_t* slot_items, WorkItem* items,
                            int32_t* item_count, int64_t* counters, cudaStream_t st);
// Q rows of every work item into an item-major image: item i occupies rows
// [128 i, 128 i + 128) (own rows, then guest rows, then zeros).
int launch_item_gather(const void* Q, int N, const int32_t* q_perm, const WorkItem* items, const int32_t* item_count,
                       size_t item_cap, void* Qimg, int num_sms, cudaStream_t st);
int launch_sparse_attn_tc(const void* Qimg, size_t item_cap, const void* Kpad, const void* Vpad, int BH, int N, int Npad,
                          int NQ, int NK, const int32_t* q_perm, const int2* segs, const float* segwA,
                          const float* segwB, const int32_t* kv_nseg, const int32_t* kv_pre, const int32_t* kv_len,
                          const WorkItem* items, const int32_t* item_count, void* O, int32_t* status, int num_sms,
                          cudaStream_t st);
int launch_sparse_attn_simt(const void* Q, const void* K, const void* V, int dtype, int BH, int N, int D, int NQ,
                            int NK, const int32_t* q_labels, const int32_t* k_perm, const int32_t* k_off,
                            const int32_t* kept_ptr, const int32_t* kept_idx, const float* bweight, void* O,
                            cudaStream_t st);

}  // namespace park
