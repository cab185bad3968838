// C ABI of libpark: argument validation, workspace carving and the launch
// sequence of park_retrieve / park_sparse_attn / park_layer.  Nothing here
// allocates or synchronises; every step is a kernel on the caller's stream.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "kernels.h"

namespace park {

static std::atomic<unsigned long long> g_launches{0};
void note_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s
static std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

// ---------------------------------------------------------------- per-kernel timing
namespace {
struct ProfRec {
    const char* name;
    cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::atomic<bool> g_prof_on{false};
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_prof_pool;
thread_local cudaEvent_t t_prof_begin = nullptr;

cudaEvent_t prof_event() {
    if (!g_prof_pool.empty()) {
        cudaEvent_t e = g_prof_pool.back();
        g_prof_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return e;
}
}  // namespace

void prof_begin(cudaStream_t st) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    t_prof_begin = prof_event();
    if (t_prof_begin) cudaEventRecord(t_prof_begin, st);
}

void prof_end(const char* name, cudaStream_t st) {
    if (!g_prof_on.load(std::memory_order_relaxed) || !t_prof_begin) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    cudaEvent_t b = prof_event();
    if (b) {
        cudaEventRecord(b, st);
        g_prof_recs.push_back({name, t_prof_begin, b});
    } else {
        g_prof_pool.push_back(t_prof_begin);
    }
    t_prof_begin = nullptr;
}

namespace {

struct Dims {
    int B, H, N, D, dtype, BH, elt;
    int T, Hg, W, nvideo;  // video grid; nvideo = T Hg W tokens precede the text tokens
};

// bf16 with D = 128: the tcgen05 kernels (assign, PAMA, attention)
inline bool tensor_path(const Dims& d) { return d.dtype == PARK_BF16 && d.D == 128; }

int check_shape(const park_shape* s, int NQ, int NK, Dims* d) {
    if (!s) return PARK_ERR_INVALID_ARG;
    if (s->B < 1 || s->H < 1 || s->T < 0 || s->Hg < 0 || s->W < 0 || s->n_text < 0 || s->D < 1)
        return PARK_ERR_INVALID_ARG;
    long long nv = (long long)s->T * s->Hg * s->W;
    long long N = nv + s->n_text;
    if (N < 1 || N > (1ll << 20)) return N < 1 ? PARK_ERR_INVALID_ARG : PARK_ERR_UNSUPPORTED;
    long long BH = (long long)s->B * s->H;
    if (BH * N >= (1ll << 31) || BH > 65535) return PARK_ERR_UNSUPPORTED;
    if (NQ < 1 || NK < 1 || NQ > N || NK > N) return PARK_ERR_INVALID_ARG;
    if (NK > 4096 || NQ > 65536) return PARK_ERR_UNSUPPORTED;
    // bf16 with D = 128 takes the tensor-core kernels; bf16 with another D, and float32,
    // take the float64 and SIMT kernels (the same certified results, slower)
    if (s->dtype != PARK_BF16 && s->dtype != PARK_F32) return PARK_ERR_INVALID_ARG;
    if (s->D % 32 != 0 || s->D > 128) return PARK_ERR_UNSUPPORTED;
    d->B = s->B;
    d->H = s->H;
    d->N = (int)N;
    d->D = s->D;
    d->dtype = s->dtype;
    d->BH = (int)BH;
    d->elt = s->dtype == PARK_BF16 ? 2 : 4;
    d->T = s->T;
    d->Hg = s->Hg;
    d->W = s->W;
    d->nvideo = (int)nv;
    return PARK_OK;
}

struct Carver {
    size_t off = 0;
    size_t take(size_t bytes) {
        size_t o = off;
        off = align_up(off + (bytes ? bytes : 1), 256);
        return o;
    }
};

constexpr int kSortChunk = 1024;
constexpr int kAttnTile = 64;     // query rows per work item, float32 path
constexpr int kAttnTileTc = 128;  // query rows per work item, tensor-core path

int metric_chunks(const Dims& d) {
    int c = (2 * 148 + d.BH - 1) / d.BH;
    int cap = (d.N + 255) / 256;
    if (c > cap) c = cap;
    if (c > 64) c = 64;
    return c < 1 ? 1 : c;
}

struct RetrievalWs {
    size_t M, Mpart, xnorm_q, xnorm_k, wop, b32, b64, w64, wmax, bmax, lfull, lcnt, hist, rho, plist,
        pcnt, kcnt, f64z, cperm, coff, mS, mP, mI, mX, mH, txt, qg, wide, tiny, total;
};

RetrievalWs plan_retrieval(const Dims& d, int NQ, int NK) {
    RetrievalWs w;
    Carver c;
    size_t BH = d.BH, N = d.N, D = d.D, Km = NQ > NK ? NQ : NK;
    size_t nchunks = (N + kSortChunk - 1) / kSortChunk;
    w.M = c.take(BH * D * D * 8);
    w.Mpart = c.take(BH * metric_chunks(d) * D * D * 8);
    w.xnorm_q = c.take(BH * N * 4);
    w.xnorm_k = c.take(BH * N * 4);
    w.wop = c.take(BH * Km * 2 * D * 2);
    w.b32 = c.take(BH * align_up(Km, 128) * 4);
    w.b64 = c.take(BH * Km * 8);
    w.w64 = c.take(BH * Km * D * 8);
    w.wmax = c.take(BH * 4);
    w.bmax = c.take(BH * 4);
    w.lfull = c.take(BH * N * 4);
    w.lcnt = c.take(BH * 4);
    w.hist = c.take(BH * Km * nchunks * 4);
    w.rho = c.take(BH * NQ * 4);
    w.plist = c.take(BH * NQ * 4);
    w.pcnt = c.take(16 * 4);
    w.wide = c.take(2 * BH * 4);  // per-head flags of Q and K: an element with |x| >= 2^16
    w.tiny = c.take(2 * BH * N);  // per-row flags of Q and K: a nonzero element with |x| < 2^-20
    w.kcnt = c.take(BH * NQ * 4);
    w.f64z = c.take(pama_f64_scratch_bytes(NK));
    w.cperm = c.take(BH * NQ * 4);
    w.coff = c.take(BH * (NQ + 1) * 4);
    const size_t Wd = (NK + 31) / 32;
    w.mS = c.take(BH * NQ * Wd * 4);
    w.mP = c.take(BH * kMergePlanes * Wd * 4);
    w.mI = c.take(7 * BH * NQ * 4);  // n, L, alive, root, best, rootf, todo
    w.mX = c.take(NQ <= kMergeMaxNQ ? BH * NQ * NQ * 4 : 0);
    w.mH = c.take(2 * BH * 4);       // done, nb
    w.txt = c.take(text_scratch_bytes(d.BH, d.N - d.nvideo, (int)Km));
    w.qg = c.take(tensor_path(d) ? BH * N * D * 2 : 0);  // Q in query-cluster order, for PAMA
    w.total = c.off;
    return w;
}


struct AttnWs {
    size_t Qimg, Kp, Vp, poff, segs, segw, segwB, kvnseg, sitems, pack, pcand, mS, mP, mI, mH, items, icnt, kvpre,
        kvlen, total;
    size_t item_cap;  // tensor-core work items at most: sum_r ceil(n_r / 128) <= ceil(N / 128) + NQ per head
    int Npad;
};

// Rows per head of the padded key layout: every key cluster rounded up to a
// multiple of 8 rows adds at most 7 rows per cluster.
int padded_rows(const Dims& d, int NK) { return (int)align_up((size_t)d.N + 7 * (size_t)NK, 8); }

AttnWs plan_attn(const Dims& d, int NQ, int NK) {
    AttnWs w;
    Carver c;
    size_t BH = d.BH, N = d.N, D = d.D;
    size_t rowbytes = D * d.elt;
    w.Npad = padded_rows(d, NK);
    w.item_cap = BH * ((N + kAttnTileTc - 1) / kAttnTileTc + (size_t)NQ);
    if (tensor_path(d)) {
        w.Qimg = c.take(w.item_cap * kAttnTileTc * rowbytes);
        w.Kp = c.take(BH * (size_t)w.Npad * rowbytes);
        w.Vp = c.take(BH * (size_t)w.Npad * rowbytes);
        w.poff = c.take(BH * (size_t)(NK + 1) * 4);
        w.segs = c.take(BH * (size_t)NQ * NK * 8);
        w.segw = c.take(BH * (size_t)NQ * NK * 4);
        w.segwB = c.take(BH * (size_t)NQ * NK * 4);
        w.kvnseg = c.take(BH * (size_t)NQ * 4);
        w.sitems = c.take(BH * (size_t)NQ * 4);
        const bool pk = NQ <= kMergeMaxNQ;  // query-tile packing (its state as in the merge)
        const size_t Wd = (NK + 31) / 32;
        w.pack = c.take(pk ? 2 * BH * (size_t)NQ * 4 : 0);
        w.pcand = c.take(pk ? BH * (size_t)NQ * kPackCandidates * 8 : 0);
        w.mS = c.take(pk ? BH * (size_t)NQ * Wd * 4 : 0);
        w.mP = c.take(pk ? BH * kMergePlanes * Wd * 4 : 0);
        w.mI = c.take(pk ? 7 * BH * (size_t)NQ * 4 : 0);
        w.mH = c.take(pk ? 2 * BH * 4 : 0);
    } else {
        w.Qimg = w.Kp = w.Vp = w.poff = w.segs = w.segw = w.segwB = w.kvnseg = w.sitems = 0;
        w.pack = w.pcand = w.mS = w.mP = w.mI = w.mH = 0;
    }
    size_t max_items = BH * ((N + kAttnTile - 1) / kAttnTile + (size_t)NQ);
    w.items = c.take(max_items * sizeof(WorkItem));
    w.icnt = c.take(16 * 4);
    w.kvpre = c.take(BH * (size_t)NQ * NK * 4);
    w.kvlen = c.take(BH * (size_t)NQ * 4);
    w.total = c.off;
    return w;
}

int num_sms_current() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
    }
    cudaGetLastError();
    return n > 0 ? n : 148;
}

template <typename P>
P* at(void* ws, size_t off) {
    return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

MergeWs merge_ws(void* ws, const RetrievalWs& w, int BH, int NQ) {
    MergeWs m;
    m.S = at<uint32_t>(ws, w.mS);
    m.P = at<uint32_t>(ws, w.mP);
    int32_t* a = at<int32_t>(ws, w.mI);
    const size_t s = (size_t)BH * NQ;
    m.n = a;
    m.L = a + s;
    m.alive = a + 2 * s;
    m.root = a + 3 * s;
    m.best = a + 4 * s;
    m.rootf = a + 5 * s;
    m.todo = a + 6 * s;
    m.inter = at<int32_t>(ws, w.mX);
    m.done = at<int32_t>(ws, w.mH);
    m.nb = m.done + BH;
    return m;
}

int memset_async(void* p, size_t n, cudaStream_t st) {
    if (cudaMemsetAsync(p, 0, n, st) != cudaSuccess) {
        cudaGetLastError();
        return PARK_ERR_CUDA;
    }
    return PARK_OK;
}

// Score-bound factors (see k_assign.cu): tensor-core fp32 accumulation of
// `terms` exact products (worst case terms * 2^-23 of sum |x_j w_j|), doubled
// because the score is bias - 2 x.w, the bf16 hi/lo split residual of M c
// (keys), and the rounding of the score itself.
float gamma_for(int terms, bool split) {
    double g = 2.0 * terms * 1.1920929e-7 * 1.01 + 2.4e-7;
    if (split) g += 2.0 * 1.52587890625e-5;
    return (float)(g * 1.05);
}

struct Side {
    const void* X;
    int K;
    void* C;
    int32_t* labels;
    int32_t* perm;
    int32_t* offsets;
    const double* M;  // null: Euclidean
    bool warm;
    int cnt_slot;
    float* xnorm;
    int Kmax;          // max(NQ, NK): leading dimension of the shared bias buffer
    int32_t* status;
    const WinGeom* win;  // non-null: HVA local-window assign
    int n_text;
    const int32_t* wide;       // per-head flags of X from the input check (general update path)
    const uint8_t* tiny_rows;  // per-row flags of X from the input check (out-of-line update rows)
};

int run_kmeans(const Dims& d, const Side& s, int iters, const RetrievalWs& w, void* ws, int64_t* counters,
               int num_sms, cudaStream_t st) {
    const bool tc = tensor_path(d);
    const int BH = d.BH, N = d.N, D = d.D, K = s.K;
    const int nchunks = (N + kSortChunk - 1) / kSortChunk;
    CentroidOps ops;
    ops.bias32 = at<float>(ws, w.b32);
    ops.bias_ld = (int)align_up((size_t)(s.Kmax), 128);
    ops.bias64 = at<double>(ws, w.b64);
    ops.w64 = s.M ? at<double>(ws, w.w64) : nullptr;
    ops.wmax = at<float>(ws, w.wmax);
    ops.bmax = at<float>(ws, w.bmax);
    if (s.M) {
        ops.w = tc ? at<uint16_t>(ws, w.wop) : nullptr;
        ops.kw = 2 * D;
    } else {
        ops.w = static_cast<const uint16_t*>(s.C);
        ops.kw = D;
    }
    Lists lists;
    lists.full_row = at<int32_t>(ws, w.lfull);
    lists.counts = at<int32_t>(ws, w.lcnt);
    if (s.win) {
        // HVA local windows: float32-certified scores against the box's centroids (text
        // tokens: against all), float64 for the rows the bound cannot decide
        ops.w = nullptr;
        if (!s.warm) PARK_CHECK(launch_local_init(s.X, d.dtype, BH, N, D, K, *s.win, s.C, st));
        for (int it = 0; it < iters; ++it) {
            PARK_CHECK(memset_async(ops.wmax, (size_t)BH * 4, st));
            PARK_CHECK(memset_async(ops.bmax, (size_t)BH * 4, st));
            PARK_CHECK(launch_centroid_prep(s.C, d.dtype, BH, K, D, s.M, ops, st));
            PARK_CHECK(launch_assign_local(s.X, d.dtype, BH, N, D, K, *s.win, s.C, ops.w64, ops.bias64, ops.wmax,
                                           ops.bmax, s.labels, counters, s.cnt_slot, st));
            if (s.n_text > 0)
                PARK_CHECK(launch_assign_text(s.X, d.dtype, BH, N, D, K, s.win->nvideo, s.C, ops.w64, ops.bias64,
                                              ops.wmax, ops.bmax, at<void>(ws, w.txt), s.labels, counters,
                                              s.cnt_slot, st));
            PARK_CHECK(launch_label_sort(s.labels, BH, N, K, at<int32_t>(ws, w.hist), nchunks, s.perm, s.offsets, st));
            PARK_CHECK(launch_update(s.X, d.dtype, BH, N, D, K, s.perm, s.offsets, s.C, s.wide, s.tiny_rows, st));
        }
        return PARK_OK;
    }
    // labels start valid (cluster 0), so that a kernel that gave up on a bounded
    // wait (status PARK_ERR_TIMEOUT) leaves nothing out of range for the later steps
    PARK_CHECK(memset_async(s.labels, (size_t)BH * N * 4, st));
    // (the row norms of the tensor-core assign bound come from the input check)
    if (!s.warm) PARK_CHECK(launch_strided_init(s.X, d.dtype, BH, N, D, K, s.C, st));
    const float gamma = gamma_for(ops.kw, s.M != nullptr);
    for (int it = 0; it < iters; ++it) {
        PARK_CHECK(memset_async(ops.wmax, (size_t)BH * 4, st));
        PARK_CHECK(memset_async(ops.bmax, (size_t)BH * 4, st));
        PARK_CHECK(memset_async(lists.counts, (size_t)BH * 4, st));
        PARK_CHECK(launch_centroid_prep(s.C, d.dtype, BH, K, D, s.M, ops, st));
        if (tc) {
            PARK_CHECK(launch_assign_tc(s.X, BH, N, K, ops, s.xnorm, gamma, s.labels, lists, s.status, num_sms, st));
            PARK_CHECK(launch_recheck(s.X, d.dtype, BH, N, D, K, s.C, ops.w64, ops.bias64, s.labels, lists, 0,
                                      num_sms, counters, s.cnt_slot, st));
        } else {
            PARK_CHECK(launch_recheck(s.X, d.dtype, BH, N, D, K, s.C, ops.w64, ops.bias64, s.labels, lists, 1,
                                      num_sms, counters, s.cnt_slot, st));
        }
        PARK_CHECK(launch_label_sort(s.labels, BH, N, K, at<int32_t>(ws, w.hist), nchunks, s.perm, s.offsets, st));
        PARK_CHECK(launch_update(s.X, d.dtype, BH, N, D, K, s.perm, s.offsets, s.C, s.wide, s.tiny_rows, st));
    }
    return PARK_OK;
}

bool retrieval_ptrs_ok(const park_retrieval* o) {
    return o && o->q_labels && o->k_labels && o->q_perm && o->k_perm && o->q_offsets && o->k_offsets &&
           o->q_centroids && o->k_centroids && o->importance && o->mask && o->kept_ptr && o->kept_idx &&
           o->counters && o->status;
}

size_t ws_bytes_for(const Dims& d, int NQ, int NK) {
    size_t a = plan_retrieval(d, NQ, NK).total, b = plan_attn(d, NQ, NK).total;
    return a > b ? a : b;
}

// Known flag bits only; with PARK_FLAG_TOPK, p is a ratio in (0, 1].
bool flags_ok(const park_retrieval* r, float p) {
    const uint32_t flags = r->flags;
    const uint32_t known = PARK_FLAG_WARM_START_Q | PARK_FLAG_WARM_START_K | PARK_FLAG_NO_QRKC |
                           PARK_FLAG_CENTROID_QUERY | PARK_FLAG_TOPK | PARK_FLAG_SIZE_PRIOR | PARK_FLAG_SIP |
                           PARK_FLAG_MERGE_Q | PARK_FLAG_LOCAL_WINDOW | PARK_FLAG_NO_TILE_PACKING;
    if (flags & ~known) return false;
    if ((flags & (PARK_FLAG_TOPK | PARK_FLAG_SIP)) && p > 1.0f) return false;
    if ((flags & PARK_FLAG_TOPK) && (flags & PARK_FLAG_SIP)) return false;
    if ((flags & PARK_FLAG_MERGE_Q) && ((flags & PARK_FLAG_SIP) || r->merge_rounds < 0 || r->merge_rounds > 64))
        return false;
    return !(flags & PARK_FLAG_SIP) || (r->sip_uniform && r->block_weight);
}

constexpr int kDefaultMergeRounds = 8;
constexpr int kMaxWindowCentroids = 256;

// Window geometry of PARK_FLAG_LOCAL_WINDOW: every extent within the grid, every
// window owning at least one query and one key centroid, at most 256 each.
int window_geometry(const park_retrieval* r, const Dims& d, int NQ, int NK, WinGeom* g) {
    if (!(r->flags & PARK_FLAG_LOCAL_WINDOW)) return PARK_OK;
    if (d.nvideo < 1 || r->window_t < 1 || r->window_h < 1 || r->window_w < 1 || r->window_t > d.T ||
        r->window_h > d.Hg || r->window_w > d.W)
        return PARK_ERR_INVALID_ARG;
    g->T = d.T;
    g->Hg = d.Hg;
    g->W = d.W;
    g->wt = r->window_t;
    g->wh = r->window_h;
    g->ww = r->window_w;
    g->nWt = (d.T + g->wt - 1) / g->wt;
    g->nWh = (d.Hg + g->wh - 1) / g->wh;
    g->nWw = (d.W + g->ww - 1) / g->ww;
    const long long nW = (long long)g->nWt * g->nWh * g->nWw;
    if (nW > NQ || nW > NK) return PARK_ERR_INVALID_ARG;
    g->nW = (int)nW;
    g->nvideo = d.nvideo;
    g->maxwin = g->wt * g->wh * g->ww;
    const int kmax = ((NQ > NK ? NQ : NK) + g->nW - 1) / g->nW;
    if (kmax > kMaxWindowCentroids) return PARK_ERR_UNSUPPORTED;
    return PARK_OK;
}

int retrieve_impl(const void* Q, const void* K, const Dims& d, int NQ, int NK, float p, int iters,
                  park_retrieval* out, void* ws, cudaStream_t st) {
    const RetrievalWs w = plan_retrieval(d, NQ, NK);
    const int num_sms = num_sms_current();
    const int BH = d.BH, N = d.N, D = d.D;
    const size_t nel = (size_t)BH * N * D;
    PARK_CHECK(memset_async(out->status, 4, st));
    PARK_CHECK(memset_async(out->counters, PARK_NUM_COUNTERS * 8, st));
    PARK_CHECK(memset_async(at<int32_t>(ws, w.pcnt), 16 * 4, st));
    int32_t* wide = at<int32_t>(ws, w.wide);
    uint8_t* tiny = at<uint8_t>(ws, w.tiny);
    PARK_CHECK(memset_async(wide, (size_t)2 * BH * 4, st));
    PARK_CHECK(memset_async(tiny, (size_t)2 * BH * N, st));
    // bf16 with D = 128: the checks also write the row norms the certified assign bound uses
    const bool norms = d.dtype == PARK_BF16 && D == 128;
    PARK_CHECK(launch_input_check(Q, nel, d.dtype, out->status, wide, (size_t)N * D, tiny, D,
                                  norms ? at<float>(ws, w.xnorm_q) : nullptr, st));
    PARK_CHECK(launch_input_check(K, nel, d.dtype, out->status, wide + BH, (size_t)N * D, tiny + (size_t)BH * N, D,
                                  norms ? at<float>(ws, w.xnorm_k) : nullptr, st));
    const uint32_t fl = out->flags;
    const bool qrkc = (fl & PARK_FLAG_NO_QRKC) == 0;
    const int select = (fl & PARK_FLAG_SIP) ? 2 : ((fl & PARK_FLAG_TOPK) ? 1 : 0);
    const int size_prior = (fl & PARK_FLAG_SIZE_PRIOR) != 0;
    const float* sip_u = select == 2 ? out->sip_uniform : nullptr;
    float* bw = select == 2 ? out->block_weight : nullptr;
    double* M = at<double>(ws, w.M);
    if (qrkc || out->metric)
        PARK_CHECK(launch_metric(Q, d.dtype, BH, N, D, at<double>(ws, w.Mpart), metric_chunks(d), M, out->metric, st));

    WinGeom geo{};
    PARK_CHECK(window_geometry(out, d, NQ, NK, &geo));
    const WinGeom* win = (fl & PARK_FLAG_LOCAL_WINDOW) ? &geo : nullptr;
    Side sq{Q, NQ, out->q_centroids, out->q_labels, out->q_perm, out->q_offsets, nullptr,
            (out->flags & PARK_FLAG_WARM_START_Q) != 0, PARK_CNT_Q_RECHECK, at<float>(ws, w.xnorm_q),
            NQ > NK ? NQ : NK, out->status, win, N - d.nvideo, wide, tiny};
    Side sk{K, NK, out->k_centroids, out->k_labels, out->k_perm, out->k_offsets, qrkc ? M : nullptr,
            (out->flags & PARK_FLAG_WARM_START_K) != 0, PARK_CNT_K_RECHECK, at<float>(ws, w.xnorm_k),
            NQ > NK ? NQ : NK, out->status, win, N - d.nvideo, wide + BH, tiny + (size_t)BH * N};
    PARK_CHECK(run_kmeans(d, sq, iters, w, ws, out->counters, num_sms, st));
    PARK_CHECK(run_kmeans(d, sk, iters, w, ws, out->counters, num_sms, st));

    int32_t* kcnt = at<int32_t>(ws, w.kcnt);
    if (fl & PARK_FLAG_CENTROID_QUERY) {
        // "w/o PAMA": each non-empty query cluster is one row, its centroid, through the float64 kernel
        int32_t* cperm = at<int32_t>(ws, w.cperm);
        int32_t* coff = at<int32_t>(ws, w.coff);
        PARK_CHECK(launch_centroid_rows(out->q_offsets, BH, NQ, cperm, coff, st));
        PARK_CHECK(launch_pama_f64(out->q_centroids, d.dtype, BH, NQ, D, NQ, NK, cperm, coff, out->k_centroids,
                                   out->k_offsets, p, select, size_prior, sip_u, bw, nullptr, nullptr, 1, num_sms,
                                   at<int32_t>(ws, w.pcnt) + 4, at<double>(ws, w.f64z), out->importance,
                                   out->importance_bound, out->mask, kcnt, out->counters, st, 1));
    } else if (tensor_path(d)) {
        // max ||c_m|| over the final key centroids, for the PAMA bound
        CentroidOps ops{nullptr, D, at<float>(ws, w.b32), (int)align_up((size_t)(NQ > NK ? NQ : NK), 128),
                        at<double>(ws, w.b64), nullptr, at<float>(ws, w.wmax), at<float>(ws, w.bmax)};
        PARK_CHECK(memset_async(ops.wmax, (size_t)BH * 4, st));
        PARK_CHECK(memset_async(ops.bmax, (size_t)BH * 4, st));
        PARK_CHECK(launch_centroid_prep(out->k_centroids, d.dtype, BH, NK, D, nullptr, ops, st));
        void* Qg = at<void>(ws, w.qg);
        PARK_CHECK(launch_gather(Q, d.dtype, BH, N, D, out->q_perm, Qg, st));
        PARK_CHECK(launch_pama_tc(Qg, BH, N, NQ, NK, out->q_perm, out->q_offsets, out->k_centroids, out->k_offsets,
                                  at<float>(ws, w.xnorm_q), size_prior, out->importance, at<float>(ws, w.rho),
                                  ops.wmax, out->status, num_sms, st));
        PARK_CHECK(launch_topp(out->importance, at<float>(ws, w.rho), BH, NQ, NK, out->q_offsets, out->k_offsets, p,
                               select, sip_u, bw, out->mask, kcnt, out->importance_bound, at<int32_t>(ws, w.plist),
                               at<int32_t>(ws, w.pcnt), st));
        PARK_CHECK(launch_pama_f64(Q, d.dtype, BH, N, D, NQ, NK, out->q_perm, out->q_offsets, out->k_centroids,
                                   out->k_offsets, p, select, size_prior, sip_u, bw, at<int32_t>(ws, w.plist),
                                   at<int32_t>(ws, w.pcnt), 0, num_sms,
                                   at<int32_t>(ws, w.pcnt) + 4, at<double>(ws, w.f64z), out->importance,
                                   out->importance_bound, out->mask, kcnt, out->counters, st));
    } else {
        PARK_CHECK(launch_pama_f64(Q, d.dtype, BH, N, D, NQ, NK, out->q_perm, out->q_offsets, out->k_centroids,
                                   out->k_offsets, p, select, size_prior, sip_u, bw, nullptr, nullptr, 1, num_sms,
                                   at<int32_t>(ws, w.pcnt) + 4,
                                   at<double>(ws, w.f64z), out->importance, out->importance_bound, out->mask, kcnt,
                                   out->counters, st));
    }
    if (fl & PARK_FLAG_MERGE_Q) {
        // HVA cluster merging; the merged clustering's permutation and centroids follow
        const int rounds = out->merge_rounds > 0 ? out->merge_rounds : kDefaultMergeRounds;
        PARK_CHECK(launch_merge(out->mask, kcnt, out->q_offsets, out->k_offsets, BH, N, NQ, NK, rounds,
                                merge_ws(ws, w, BH, NQ), out->q_labels, num_sms, st));
        const int nchunks = (N + kSortChunk - 1) / kSortChunk;
        PARK_CHECK(launch_label_sort(out->q_labels, BH, N, NQ, at<int32_t>(ws, w.hist), nchunks, out->q_perm,
                                     out->q_offsets, st));
        PARK_CHECK(launch_update(Q, d.dtype, BH, N, D, NQ, out->q_perm, out->q_offsets, out->q_centroids, wide, tiny,
                                 st));
    }
    PARK_CHECK(launch_kept_csr(out->mask, kcnt, BH, NQ, NK, out->kept_ptr, out->kept_idx, out->counters, st));
    return PARK_OK;
}

int attn_impl(const void* Q, const void* K, const void* V, const Dims& d, int NQ, int NK, const park_retrieval* r,
              void* O, void* ws, cudaStream_t st) {
    const AttnWs w = plan_attn(d, NQ, NK);
    const int BH = d.BH, N = d.N, D = d.D;
    const bool tc = tensor_path(d);
    PARK_CHECK(launch_input_check(V, (size_t)BH * N * D, d.dtype, r->status, nullptr, (size_t)N * D, nullptr, D,
                                  nullptr, st));
    PARK_CHECK(memset_async(r->counters + PARK_CNT_KEPT_PAIRS, 3 * sizeof(int64_t), st));
    int32_t* icnt = at<int32_t>(ws, w.icnt);
    PARK_CHECK(memset_async(icnt, 16 * 4, st));
    const float* bw = (r->flags & PARK_FLAG_SIP) ? r->block_weight : nullptr;  // SIP weights
    if (!tc) {
        PARK_CHECK(launch_attn_schedule(BH, NQ, NK, r->q_offsets, r->k_offsets, r->kept_ptr, r->kept_idx,
                                        at<int32_t>(ws, w.kvpre), at<int32_t>(ws, w.kvlen), at<WorkItem>(ws, w.items),
                                        icnt, r->counters, kAttnTile, 0, nullptr, 0, nullptr, nullptr, nullptr, st));
        return launch_sparse_attn_simt(Q, K, V, d.dtype, BH, N, D, NQ, NK, r->q_labels, r->k_perm, r->k_offsets,
                                       r->kept_ptr, r->kept_idx, bw, O, st);
    }
    const int num_sms = num_sms_current();
    void* Qimg = at<void>(ws, w.Qimg);
    void* Kp = at<void>(ws, w.Kp);
    void* Vp = at<void>(ws, w.Vp);
    int32_t* poff = at<int32_t>(ws, w.poff);
    int2* segs = at<int2>(ws, w.segs);
    float* segwA = at<float>(ws, w.segw);
    float* segwB = at<float>(ws, w.segwB);
    int32_t* kvnseg = at<int32_t>(ws, w.kvnseg);
    WorkItem* items = at<WorkItem>(ws, w.items);
    PARK_CHECK(launch_kv_pad_gather(K, V, BH, N, NK, w.Npad, r->k_perm, r->k_labels, r->k_offsets, poff, Kp, Vp, st));
    // query-tile packing: a guest's last tile shares its host's single tile (exact: every row keeps
    // only its own cluster's key blocks)
    int32_t* pack_host = nullptr;
    int32_t* pack_guest = nullptr;
    if (!(r->flags & PARK_FLAG_NO_TILE_PACKING) && NQ <= kMergeMaxNQ) {
        pack_host = at<int32_t>(ws, w.pack);
        pack_guest = pack_host + (size_t)BH * NQ;
        MergeWs m;
        m.S = at<uint32_t>(ws, w.mS);
        m.P = at<uint32_t>(ws, w.mP);
        m.inter = nullptr;
        int32_t* a = at<int32_t>(ws, w.mI);
        const size_t sN = (size_t)BH * NQ;
        m.n = a;
        m.L = a + sN;
        m.alive = a + 2 * sN;
        m.root = a + 3 * sN;
        m.best = a + 4 * sN;
        m.rootf = a + 5 * sN;
        m.todo = a + 6 * sN;
        m.done = at<int32_t>(ws, w.mH);
        m.nb = m.done + BH;
        PARK_CHECK(launch_pack_pairs(BH, NQ, NK, r->mask, r->q_offsets, r->k_offsets, m, at<int2>(ws, w.pcand),
                                     pack_host, pack_guest, st));
    }
    PARK_CHECK(launch_attn_schedule_tc(BH, NQ, NK, w.Npad, r->q_offsets, r->k_offsets, r->mask, bw, poff, pack_host,
                                       pack_guest, at<int32_t>(ws, w.kvpre), at<int32_t>(ws, w.kvlen), kvnseg, segs,
                                       segwA, segwB, at<int32_t>(ws, w.sitems), items, icnt, r->counters, st));
    PARK_CHECK(launch_item_gather(Q, N, r->q_perm, items, icnt, w.item_cap, Qimg, num_sms, st));
    PARK_CHECK(launch_sparse_attn_tc(Qimg, w.item_cap, Kp, Vp, BH, N, w.Npad, NQ, NK, r->q_perm, segs, segwA, segwB,
                                     kvnseg, at<int32_t>(ws, w.kvpre), at<int32_t>(ws, w.kvlen), items, icnt, O,
                                     r->status, num_sms, st));
    return PARK_OK;
}

}  // namespace
}  // namespace park

using namespace park;

extern "C" {

int park_workspace_size(const park_shape* shape, int NQ, int NK, size_t* bytes) {
    Dims d;
    if (!bytes) return PARK_ERR_INVALID_ARG;
    PARK_CHECK(check_shape(shape, NQ, NK, &d));
    *bytes = ws_bytes_for(d, NQ, NK);
    return PARK_OK;
}

int park_retrieve(const void* Q, const void* K, const park_shape* shape, int NQ, int NK, float p, int iters,
                  park_retrieval* out, void* ws, size_t ws_bytes, void* stream) {
    Dims d;
    PARK_CHECK(check_shape(shape, NQ, NK, &d));
    if (!Q || !K || !ws || !retrieval_ptrs_ok(out)) return PARK_ERR_INVALID_ARG;
    if (!(p > 0.0f) || !std::isfinite(p) || iters < 1) return PARK_ERR_INVALID_ARG;
    if (!flags_ok(out, p)) return PARK_ERR_INVALID_ARG;
    if ((out->flags & PARK_FLAG_MERGE_Q) && NQ > kMergeMaxNQ) return PARK_ERR_UNSUPPORTED;
    WinGeom geo;
    PARK_CHECK(window_geometry(out, d, NQ, NK, &geo));
    if (ws_bytes < ws_bytes_for(d, NQ, NK)) return PARK_ERR_WORKSPACE;
    return retrieve_impl(Q, K, d, NQ, NK, p, iters, out, ws, static_cast<cudaStream_t>(stream));
}

int park_sparse_attn(const void* Q, const void* K, const void* V, const park_shape* shape, int NQ, int NK,
                     const park_retrieval* r, void* O, void* ws, size_t ws_bytes, void* stream) {
    Dims d;
    PARK_CHECK(check_shape(shape, NQ, NK, &d));
    if (!Q || !K || !V || !O || !ws || !retrieval_ptrs_ok(r)) return PARK_ERR_INVALID_ARG;
    if ((r->flags & PARK_FLAG_SIP) && !r->block_weight) return PARK_ERR_INVALID_ARG;
    if (ws_bytes < ws_bytes_for(d, NQ, NK)) return PARK_ERR_WORKSPACE;
    return attn_impl(Q, K, V, d, NQ, NK, r, O, ws, static_cast<cudaStream_t>(stream));
}

int park_layer(const void* Q, const void* K, const void* V, const park_shape* shape, int NQ, int NK, float p,
               int iters, void* O, park_retrieval* out, void* ws, size_t ws_bytes, void* stream) {
    Dims d;
    PARK_CHECK(check_shape(shape, NQ, NK, &d));
    if (!Q || !K || !V || !O || !ws || !retrieval_ptrs_ok(out)) return PARK_ERR_INVALID_ARG;
    if (!(p > 0.0f) || !std::isfinite(p) || iters < 1) return PARK_ERR_INVALID_ARG;
    if (!flags_ok(out, p)) return PARK_ERR_INVALID_ARG;
    if ((out->flags & PARK_FLAG_MERGE_Q) && NQ > kMergeMaxNQ) return PARK_ERR_UNSUPPORTED;
    WinGeom geo;
    PARK_CHECK(window_geometry(out, d, NQ, NK, &geo));
    if (ws_bytes < ws_bytes_for(d, NQ, NK)) return PARK_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    PARK_CHECK(retrieve_impl(Q, K, d, NQ, NK, p, iters, out, ws, st));
    return attn_impl(Q, K, V, d, NQ, NK, out, O, ws, st);
}

const char* park_status_string(int code) {
    switch (code) {
        case PARK_OK: return "ok";
        case PARK_ERR_INVALID_ARG: return "invalid argument";
        case PARK_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case PARK_ERR_WORKSPACE: return "workspace too small";
        case PARK_ERR_CUDA: return "CUDA launch failed";
        case PARK_ERR_RANGE: return "input outside the range precondition (0 or 2^-40 <= |x| < 2^40, finite)";
        case PARK_ERR_TIMEOUT: return "a bounded device wait ran out";
        default: return "unknown status";
    }
}

uint64_t park_launch_count(void) { return (uint64_t)g_launches.load(); }

int park_profile_enable(int on) {
    g_prof_on.store(on != 0);
    return PARK_OK;
}

int park_profile_collect(park_kernel_time* out, int cap, int* n) {
    if (!n || cap < 0 || (cap > 0 && !out)) return PARK_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    int count = 0, rc = PARK_OK;
    for (const ProfRec& r : g_prof_recs) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
            cudaGetLastError();
            rc = PARK_ERR_CUDA;
        }
        int slot = -1;
        for (int i = 0; i < count; ++i)
            if (std::strcmp(out[i].name, r.name) == 0) slot = i;
        if (slot < 0 && count < cap) {
            slot = count++;
            std::memset(&out[slot], 0, sizeof(park_kernel_time));
            std::strncpy(out[slot].name, r.name, sizeof(out[slot].name) - 1);
        }
        if (slot >= 0) {
            out[slot].total_ms += ms;
            out[slot].launches += 1;
        }
        g_prof_pool.push_back(r.a);
        g_prof_pool.push_back(r.b);
    }
    g_prof_recs.clear();
    *n = count;
    return rc;
}

int park_version(void) { return 200; }

int park_set_wait_limit_ns(uint64_t ns) {
    g_wait_ns.store(ns ? ns : kDefaultWaitNs, std::memory_order_relaxed);
    return PARK_OK;
}

}  // extern "C"
