// park_qrkc_metric_static: the QRKC metric M = (1/N) sum_i q_i q_i^T without any
// caller workspace.
//
// Who needs it: callers that cannot allocate device memory at the point where
// they need the metric -- for example code that runs while a CUDA graph is
// being captured (cudaMalloc is not a capturable operation), or a host
// framework that hands a plug-in only its input and output buffers and owns
// every allocation itself.  park_retrieve takes its scratch from the caller's
// workspace; this entry point takes it from a fixed array compiled into the
// library instead, so the caller passes nothing but Q and the output M.
//
// The scratch is a file-scope __device__ array of kStaticScratchBytes
// (16 MiB).  Every GPU that loads the library holds it until the process exits.
// It holds the per-chunk partial sums of the metric: one D x D float64 matrix
// per (head, row chunk), so at most 16 MiB / (8 D^2) partials (128 at D = 128):
// the number of row chunks per head is reduced to fit, and shapes with more
// than that many heads are rejected with PARK_ERR_UNSUPPORTED before any work
// is enqueued.
//
// Host code cannot use the array's name as a device address (it is a host-side
// stand-in), so on the first call on each device, with that device current,
// the entry point looks the address up once with cudaGetSymbolAddress and
// caches it; make that first call before any stream capture.  Every call
// shares the one array: calls that overlap on the GPU (different streams, or
// several host threads) race on it.  Each call writes every entry of the
// partials that its reduction reads (the upper-triangle 8 x 8 blocks of each
// D x D partial), so nothing has to start at zero.  No cudaMalloc, cudaFree or
// allocating library routine is called.
#include <mutex>

#include "kernels.h"

namespace park {

constexpr size_t kStaticScratchBytes = 16u << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up once).
int static_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return PARK_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return PARK_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (!g_static_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return PARK_ERR_CUDA;
        }
        g_static_ptr[dev] = p;
    }
    *out = g_static_ptr[dev];
    return PARK_OK;
}
}  // namespace

}  // namespace park

using namespace park;

extern "C" int park_qrkc_metric_static(const void* Q, const park_shape* shape, double* M, void* stream) {
    if (!Q || !M || !shape) return PARK_ERR_INVALID_ARG;
    const park_shape* s = shape;
    if (s->B < 1 || s->H < 1 || s->T < 0 || s->Hg < 0 || s->W < 0 || s->n_text < 0) return PARK_ERR_INVALID_ARG;
    const long long N = (long long)s->T * s->Hg * s->W + s->n_text;
    const long long BH = (long long)s->B * s->H;
    if (N < 1) return PARK_ERR_INVALID_ARG;
    if (N > (1ll << 20) || BH * N >= (1ll << 31)) return PARK_ERR_UNSUPPORTED;
    if (s->dtype == PARK_BF16) {
        if (s->D != 128) return PARK_ERR_UNSUPPORTED;
    } else if (s->dtype == PARK_F32) {
        if (s->D % 32 != 0 || s->D > 128 || s->D < 32) return PARK_ERR_UNSUPPORTED;
    } else {
        return PARK_ERR_INVALID_ARG;
    }
    const size_t per_partial = (size_t)s->D * s->D * sizeof(double);
    const long long capacity = (long long)(kStaticScratchBytes / per_partial);
    if (BH > capacity) return PARK_ERR_UNSUPPORTED;  // not even one row chunk per head fits
    // row chunks per head: as park_retrieve uses (about two CTAs per SM overall),
    // reduced so that BH * chunks partials fit in the array
    long long chunks = (2 * 148 + BH - 1) / BH;
    const long long cap_rows = (N + 255) / 256;
    if (chunks > cap_rows) chunks = cap_rows;
    if (chunks > 64) chunks = 64;
    if (chunks > capacity / BH) chunks = capacity / BH;
    if (chunks < 1) chunks = 1;
    void* scratch = nullptr;
    PARK_CHECK(static_scratch(&scratch));
    return launch_metric(Q, s->dtype, (int)BH, (int)N, s->D, static_cast<double*>(scratch), (int)chunks, M, nullptr,
                         static_cast<cudaStream_t>(stream));
}
