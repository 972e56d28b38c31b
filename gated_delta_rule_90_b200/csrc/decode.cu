// Single-token decode step of the gated delta rule, in place on the fp32 state.
//
// The token update ("Linear Attention, Visualized", DeltaNet / Recurrent form,
// with the decay of "Gated DeltaNet (GDN) / Decay also changes the correction
// rows" or, per channel, "Kimi Delta Attention (KDA)"), column convention:
//     S' = S D;  p = S' k;  u = beta (v - p);  S <- S' + u k^T;  o = S q.
// Every row i of S (d_k contiguous floats) evolves on its own given the token:
//     s_i <- a . s_i (a = decay, scalar or per key channel)
//     p_i = s_i . k,  r_i = s_i . q,  u_i = beta (v_i - p_i)
//     s_i <- s_i + u_i k,   o_i = r_i + u_i (k . q).
// So one warp owns a row at a time (32 lanes x d_k/32 floats, 128-bit loads),
// reduces the two dot products with shuffles and writes the row back: the
// state is read once and written once, which is the whole HBM cost of a step.
//
// With DEC (Gated DeltaNet-2, "Gated DeltaNet-2, and the gate that was doing
// two jobs", section "What decoupling actually means here") the erase vector
// e = b . k reads the row and the write gate scales the value:
//     p_i = s_i . e,  u_i = w_i v_i - p_i,  s_i <- s_i + u_i k.
#include "common.cuh"

namespace gdr {

template <int VEC>
struct VecF;
template <>
struct VecF<4> {
    using T = float4;
    __device__ __forceinline__ static void unpack(const T &x, float *f) {
        f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
    }
    __device__ __forceinline__ static T pack(const float *f) { return make_float4(f[0], f[1], f[2], f[3]); }
};
template <>
struct VecF<2> {
    using T = float2;
    __device__ __forceinline__ static void unpack(const T &x, float *f) { f[0] = x.x; f[1] = x.y; }
    __device__ __forceinline__ static T pack(const float *f) { return make_float2(f[0], f[1]); }
};

constexpr int kDecodeThreads = 128;  // 4 warps, each owns d_v/4 rows of one head
constexpr int kRowsInFlight = 8;     // rows a warp loads before using any

template <typename Tin, int DK, bool CHANNEL, bool DEC>
__global__ void __launch_bounds__(kDecodeThreads)
decode_step_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                   const float *__restrict__ g, const float *__restrict__ beta,
                   const float *__restrict__ eg, const float *__restrict__ wg,
                   float *__restrict__ S, Tin *__restrict__ out, int dv, long long nheads,
                   unsigned int *err) {
    constexpr int VEC = DK / 32;
    using V = VecF<VEC>;
    const size_t head = blockIdx.x;  // flattened (sequence, head)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (kChecked) {  // checked build: this head's slices of every buffer, whole row batches
        const long long hd = (long long)head;
        if (!(chk_span(hd * DK, DK, nheads * DK, err) &&                              // q, k, g, eg
              chk_span(hd * dv, dv, nheads * dv, err) &&                              // v, out, wg
              chk_span(hd * dv * DK, (long long)dv * DK, nheads * dv * DK, err) &&    // S
              chk_span(hd, 1, nheads, err) &&                                          // g, beta
              chk_true(dv % (4 * kRowsInFlight) == 0, err)))
            return;
    }

    float kk[VEC], qq[VEC], aa[VEC], ee[VEC];  // ee: the reading direction
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
        kk[j] = ld_in(k, head * DK + lane * VEC + j);
        qq[j] = ld_in(q, head * DK + lane * VEC + j);
        ee[j] = DEC ? kk[j] * eg[head * DK + lane * VEC + j] : kk[j];
    }
    if (CHANNEL) {
#pragma unroll
        for (int j = 0; j < VEC; ++j) aa[j] = expf(g[head * DK + lane * VEC + j]);
    } else {
        const float a = expf(g[head]);
#pragma unroll
        for (int j = 0; j < VEC; ++j) aa[j] = a;
    }
    float kq = 0.f;
#pragma unroll
    for (int j = 0; j < VEC; ++j) kq = fmaf(kk[j], qq[j], kq);
#pragma unroll
    for (int off = 16; off; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    const float b = DEC ? 1.f : beta[head];

    const int rpw = dv >> 2;  // rows per warp (dv is a multiple of 32)
    const int row0 = warp * rpw;
    float *Sh = S + head * (size_t)dv * DK;
    const Tin *vh = v + head * (size_t)dv;
    Tin *oh = out + head * (size_t)dv;
    float my_o = 0.f;

    for (int r0 = 0; r0 < rpw; r0 += kRowsInFlight) {
        typename V::T raw[kRowsInFlight];
        float vi[kRowsInFlight];
#pragma unroll
        for (int j = 0; j < kRowsInFlight; ++j) {
            const int row = row0 + r0 + j;
            raw[j] = __ldcs(reinterpret_cast<const typename V::T *>(Sh + (size_t)row * DK) + lane);
            vi[j] = ld_in(vh, row);
            if (DEC) vi[j] *= wg[head * (size_t)dv + row];
        }
#pragma unroll
        for (int j = 0; j < kRowsInFlight; ++j) {
            float s[VEC];
            V::unpack(raw[j], s);
            float p = 0.f, r = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                s[e] *= aa[e];
                p = fmaf(s[e], ee[e], p);
                r = fmaf(s[e], qq[e], r);
            }
#pragma unroll
            for (int off = 16; off; off >>= 1) {
                p += __shfl_xor_sync(0xffffffffu, p, off);
                r += __shfl_xor_sync(0xffffffffu, r, off);
            }
            const float u = b * (vi[j] - p);
#pragma unroll
            for (int e = 0; e < VEC; ++e) s[e] = fmaf(u, kk[e], s[e]);
            const int row = row0 + r0 + j;
            __stcs(reinterpret_cast<typename V::T *>(Sh + (size_t)row * DK) + lane, V::pack(s));
            const float o = fmaf(u, kq, r);
            const int jl = r0 + j;  // row index within this warp's rows
            if ((jl & 31) == lane) my_o = o;
            if ((jl & 31) == 31 || jl == rpw - 1) {
                if (lane <= (jl & 31)) st_out(oh, row0 + (jl & ~31) + lane, my_o);
            }
        }
    }
}

}  // namespace gdr

using namespace gdr;

template <typename Tin, int DK, bool CH, bool DEC = false>
static cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, float *S, void *out, int N, int H, int dv,
                                 cudaStream_t st, const float *eg = nullptr,
                                 const float *wg = nullptr) {
    const unsigned int blocks = (unsigned int)((size_t)N * H);
    decode_step_kernel<Tin, DK, CH, DEC><<<blocks, kDecodeThreads, 0, st>>>(
        (const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta, eg, wg, S, (Tin *)out, dv,
        (long long)N * H, kChecked ? gdr_host::device_error_word() : nullptr);
    return cudaGetLastError();
}

namespace gdr_host {
cudaError_t decode_dispatch(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float *S, void *out, int N, int H, int dk, int dv,
                            gdr_dtype dtype, gdr_gate gate, cudaStream_t st) {
    const bool ch = gate == GDR_GATE_PER_KEY_CHANNEL;
#define GDR_DEC(T, DK)                                                                        \
    return ch ? launch_decode<T, DK, true>(q, k, v, g, beta, S, out, N, H, dv, st)            \
              : launch_decode<T, DK, false>(q, k, v, g, beta, S, out, N, H, dv, st)
    if (dtype == GDR_BF16) {
        if (dk == 128) GDR_DEC(__nv_bfloat16, 128);
        GDR_DEC(__nv_bfloat16, 64);
    }
    if (dk == 128) GDR_DEC(float, 128);
    GDR_DEC(float, 64);
#undef GDR_DEC
}
// Gated DeltaNet-2 step: erase gate eg [N, H, d_k], write gate wg [N, H, d_v].
cudaError_t decode_gdn2_dispatch(const void *q, const void *k, const void *v, const float *g,
                                 const float *eg, const float *wg, float *S, void *out, int N,
                                 int H, int dk, int dv, gdr_dtype dtype, gdr_gate gate,
                                 cudaStream_t st) {
    const bool ch = gate == GDR_GATE_PER_KEY_CHANNEL;
#define GDR_DEC2(T, DK)                                                                          \
    return ch ? launch_decode<T, DK, true, true>(q, k, v, g, nullptr, S, out, N, H, dv, st, eg,  \
                                                 wg)                                             \
              : launch_decode<T, DK, false, true>(q, k, v, g, nullptr, S, out, N, H, dv, st, eg, \
                                                  wg)
    if (dtype == GDR_BF16) {
        if (dk == 128) GDR_DEC2(__nv_bfloat16, 128);
        GDR_DEC2(__nv_bfloat16, 64);
    }
    if (dk == 128) GDR_DEC2(float, 128);
    GDR_DEC2(float, 64);
#undef GDR_DEC2
}
}  // namespace gdr_host
