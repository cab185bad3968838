// Shared device helpers of libpark (no method arithmetic beyond exact
// conversions): status word, exact fixed-point conversion of inputs, correctly
// rounded conversions, warp reductions, launch accounting.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "park.h"

namespace park {

// ---------------------------------------------------------------- host side
void note_launch(int n = 1);  // counts kernels for park_launch_count()
// Limit of every bounded device wait on the hot path, in ns (park_set_wait_limit_ns).
uint64_t wait_limit_ns();
// Per-kernel event timing (park_profile_enable): begin before a launch, end
// (with the kernel's name) right after it, on the launch stream.
void prof_begin(cudaStream_t st);
void prof_end(const char* name, cudaStream_t st);

#define PARK_TRY_LAUNCH(name, st)                                \
    do {                                                         \
        ::park::prof_end(name, st);                              \
        ::park::note_launch();                                   \
        if (cudaPeekAtLastError() != cudaSuccess) {              \
            cudaGetLastError();                                  \
            return PARK_ERR_CUDA;                                \
        }                                                        \
    } while (0)

#define PARK_CHECK(x)                     \
    do {                                  \
        int _rc = (x);                    \
        if (_rc != PARK_OK) return _rc;   \
    } while (0)

static inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- element traits
struct bf16_t {
    uint16_t bits;
};

template <typename T>
struct Elem;

template <>
struct Elem<bf16_t> {
    static constexpr int bytes = 2;
    static constexpr int dtype = PARK_BF16;
    __device__ static inline double to_double(const bf16_t* p, int j) {
        return (double)__uint_as_float(((uint32_t)p[j].bits) << 16);
    }
    __device__ static inline float to_float(const bf16_t* p, int j) {
        return __uint_as_float(((uint32_t)p[j].bits) << 16);
    }
    // biased exponent (IEEE single layout) of element j
    __device__ static inline int biased_exp(uint32_t bits) { return (bits >> 7) & 0xFF; }
};

template <>
struct Elem<float> {
    static constexpr int bytes = 4;
    static constexpr int dtype = PARK_F32;
    __device__ static inline double to_double(const float* p, int j) { return (double)p[j]; }
    __device__ static inline float to_float(const float* p, int j) { return p[j]; }
    __device__ static inline int biased_exp(uint32_t bits) { return (bits >> 23) & 0xFF; }
};

// ---------------------------------------------------------------- status
__device__ inline void set_status(int32_t* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Range precondition: x == 0, or finite with 2^-40 <= |x| < 2^40
// (biased exponent 87..166 in the IEEE single layout that bf16 shares).
constexpr int kRangeExpMin = 87, kRangeExpMax = 166;
__device__ inline bool in_range_exp(int e, uint32_t magnitude_bits) {
    return magnitude_bits == 0 || (e >= kRangeExpMin && e <= kRangeExpMax);
}

// ---------------------------------------------------------------- fixed point
// Exact centroid sums: every element in range is an integer multiple of 2^-64
// (bf16: 8-bit significand, ulp >= 2^-47; float32: 24-bit significand, ulp >=
// 2^-63) below 2^40, so F = x * 2^64 is an integer with |F| < 2^104, and a sum
// of up to 2^20 of them fits a signed 128-bit integer (hi * 2^64 + lo, two's
// complement).  Integer sums do not depend on the order of the terms.
__device__ inline void acc128_add(unsigned long long& lo, long long& hi, unsigned long long a_lo, long long a_hi) {
    const unsigned long long n = lo + a_lo;
    hi += a_hi + (long long)(n < lo);
    lo = n;
}

// Adds F = x * 2^64 for the element with IEEE-single-layout bits `u` (a bf16
// element passed as its bits << 16): x = (-1)^s m 2^(e - 150) with the 24-bit
// significand m, so F = m << (e - 86), a shift of 1..80 inside the range.
// Zero adds nothing; elements outside the range (reported by the input check)
// are clamped, not summed exactly.
__device__ inline void fixed64_add(unsigned long long& lo, long long& hi, uint32_t u) {
    const int e = (u >> 23) & 0xFF;
    if (e == 0) return;
    const unsigned long long m = 0x800000ull | (u & 0x7FFFFFull);
    int sh = e - 86;
    sh = sh < 0 ? 0 : (sh > 80 ? 80 : sh);
    unsigned long long a_lo, a_hi;
    if (sh >= 64) {
        a_lo = 0ull;
        a_hi = m << (sh - 64);
    } else {
        a_lo = m << sh;
        a_hi = sh == 0 ? 0ull : (m >> (64 - sh));
    }
    if (u & 0x80000000u) {  // two's complement negation of the 128-bit value
        a_lo = ~a_lo + 1ull;
        a_hi = ~a_hi + (a_lo == 0ull ? 1ull : 0ull);
    }
    acc128_add(lo, hi, a_lo, (long long)a_hi);
}

// Correctly rounded (nearest, ties to even) conversion of the signed 128-bit
// integer hi * 2^64 + lo (two's complement) to double.
__device__ inline double i128_to_double_rn(long long hi, unsigned long long lo) {
    bool neg = hi < 0;
    unsigned long long uh = (unsigned long long)hi, ul = lo;
    if (neg) {  // negate the 128-bit value
        ul = ~ul + 1ull;
        uh = ~uh + (ul == 0ull ? 1ull : 0ull);
    }
    double r;
    if (uh == 0ull) {
        r = __ull2double_rn(ul);
    } else {
        int lz = __clzll((long long)uh);
        int sh = 64 - lz;  // bits of uh; value = (uh:ul) >> sh fits in 64 bits
        unsigned long long top, dropped;
        if (sh == 64) {
            top = uh;
            dropped = ul;
        } else {
            top = (uh << lz) | (ul >> sh);
            dropped = ul & ((1ull << sh) - 1ull);
        }
        // top has its leading bit at position 63: 53 kept bits, 11 guard bits.
        // Folding the dropped bits into the lowest guard bit (sticky) keeps the
        // nearest-even decision of the 64-bit conversion exact.
        top |= (dropped != 0ull) ? 1ull : 0ull;
        r = ldexp(__ull2double_rn(top), sh);
    }
    return neg ? -r : r;
}

// Round a double to bf16 (nearest, ties to even) directly, without passing
// through float.  Finite inputs whose magnitude is at most 2^127; values
// below the bf16 normal range (2^-126) flush to zero (never reached by means of
// inputs meeting the range precondition, which are >= 2^-67 or 0).
__device__ inline uint16_t double_to_bf16_bits(double x) {
    unsigned long long u = (unsigned long long)__double_as_longlong(x);
    unsigned long long sign = u >> 63;
    int e = (int)((u >> 52) & 0x7FF);
    int ebf = e - 1023 + 127;
    if (e == 0 || ebf <= 0) return (uint16_t)(sign << 15);
    unsigned long long mant = (u & 0xFFFFFFFFFFFFFull) | (1ull << 52);
    unsigned long long keep = mant >> 45;  // 8 significant bits
    unsigned long long rem = mant & ((1ull << 45) - 1ull);
    const unsigned long long half = 1ull << 44;
    if (rem > half || (rem == half && (keep & 1ull))) keep++;
    if (keep == 256ull) {
        keep = 128ull;
        ebf++;
    }
    if (ebf >= 255) return (uint16_t)((sign << 15) | 0x7F80u);
    return (uint16_t)((sign << 15) | ((unsigned long long)ebf << 7) | (keep & 0x7Full));
}

// ---------------------------------------------------------------- warp helpers
__device__ inline int warp_sum_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ inline float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ inline double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ inline float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ inline double warp_max(double v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// atomic max for non-negative floats (bit patterns order like integers)
__device__ inline void atomic_max_nonneg(float* addr, float v) {
    atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
}

// Round a float up by a few ulps (used to make computed bounds conservative).
__device__ inline float round_up_f(float v) { return v * (1.0f + 1.0e-6f) + 1.0e-30f; }

}  // namespace park
