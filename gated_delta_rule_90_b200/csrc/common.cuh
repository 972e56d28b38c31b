// Shared device helpers of the gated delta rule kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr.h"

namespace gdr {

// Bits of the device error word (see gdr_device_status): a bounded wait
// expired; a factorisation met a non-positive pivot (a negative writing
// strength, or NaN input); a bounds guard of the checked build refused an access.
enum : unsigned int { kErrTimeout = 1u, kErrNumeric = 2u, kErrBounds = 4u };

// ---------------------------------------------------------------- checked build
// Compiled with -DGDR_CHECK, every kernel checks, before it touches memory,
// the spans of each global buffer that its CTA will read or write (and the
// coordinates of its TMA copies) against the extents the entry point was
// called with.  A miss sets kErrBounds in the device error word and the CTA
// returns without touching anything, before any barrier, TMEM allocation or
// copy, so the kernel ends normally and gdr_device_status reports
// GDR_ERR_BOUNDS.  In the normal build the guards compile to nothing.
#ifdef GDR_CHECK
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

// Is [first, first + count) inside [0, extent)?  (count = 0 always passes.)
__device__ __forceinline__ bool chk_span(long long first, long long count, long long extent,
                                         unsigned int *err) {
    if (!kChecked || count <= 0) return true;
    if (first >= 0 && first + count <= extent) return true;
    if (err) atomicOr(err, kErrBounds);
    return false;
}
// A shape condition the kernel's index arithmetic relies on.
__device__ __forceinline__ bool chk_true(bool cond, unsigned int *err) {
    if (!kChecked || cond) return true;
    if (err) atomicOr(err, kErrBounds);
    return false;
}
// A tiled TMA copy of a box_x x box_y box at (x, y) of a tensor with x_extent
// elements per row (element size esz bytes) and `rows` rows: x must be >= 0
// with x * esz a multiple of 16 (an unaligned x is an illegal instruction), the
// box must start inside the tensor, and y >= 0 (loads may run past the end,
// which the copy fills with zeros; stores are clipped there).
__device__ __forceinline__ bool chk_tma(long long x, long long y, int esz, long long x_extent,
                                        long long rows, unsigned int *err) {
    if (!kChecked) return true;
    if (x >= 0 && (x * esz) % 16 == 0 && x < x_extent && y >= 0 && y < rows) return true;
    if (err) atomicOr(err, kErrBounds);
    return false;
}

// Token-storage loads/stores: fp32 or bf16, converted to/from fp32.
__device__ __forceinline__ float ld_in(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld_in(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st_out(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16 *p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// Sequence bounds [t0, t1) of sequence s, in token rows of the [B*T] view.
// Packed offsets are clamped into [0, T_total] and made non-decreasing so a
// malformed array can never send a kernel out of bounds.
__device__ __forceinline__ void seq_bounds(const int32_t *cu, int s, int T, int T_total,
                                           long &t0, long &t1) {
    if (cu) {
        int a = cu[s], b = cu[s + 1];
        a = a < 0 ? 0 : (a > T_total ? T_total : a);
        b = b < a ? a : (b > T_total ? T_total : b);
        t0 = a;
        t1 = b;
    } else {
        t0 = (long)s * T;
        t1 = t0 + T;
    }
}

// bf16 <-> fp32 in groups of 8 (one 16-byte vector); ld8 reads 8 floats from
// a 16-byte-aligned address.
__device__ __forceinline__ void unpack8(const uint4 &u, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ void ld8(const float *p, float *f) {
    const float4 x = reinterpret_cast<const float4 *>(p)[0], y = reinterpret_cast<const float4 *>(p)[1];
    f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
    f[4] = y.x; f[5] = y.y; f[6] = y.z; f[7] = y.w;
}
__device__ __forceinline__ uint4 pack8(const float *f) {
    uint4 u;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return u;
}

}  // namespace gdr

// Host-side launch helpers shared by the translation units.
namespace gdr_host {
// Address of the device error word on the current device (cached per device).
unsigned int *device_error_word();
// Launch accounting: call prof_begin before and prof_end after a launch of
// kernel `id` on stream `st` (events are recorded only while timing is on).
struct ProfToken {
    int id;
    int slot;
};
ProfToken prof_begin(int id, cudaStream_t st);
void prof_end(ProfToken tok, cudaStream_t st);
}  // namespace gdr_host
