// Gated DeltaProduct (GDP) forward, run as Gated DeltaNet over a virtual sequence.
//
// "Linear Attention, Visualized", section "Gated Delta Product (GDP)": every
// real token t applies n_h generalised Householder substeps (k_tj, v_tj,
// beta_tj), j = 1..n_h, after one decay a_t, and reads the state with q_t after
// the last substep.  Section "GDP as GDN over a virtual sequence": flatten
// (t, j) into m = n_h (t - 1) + j with
//     k~_m = k_tj, v~_m = v_tj, beta~_m = beta_tj,
//     a~_m = a_t for j = 1, else 1   (log-decay g~_m = g_t for j = 1, else 0),
//     q~_m = q_t for j = n_h, else 0,
// run the GDN (or per-channel) recurrence over the n n_h virtual steps and keep
// every n_h-th output.
//
// With k, v laid out [B, T, n_h, H, d] and beta [B, T, n_h, H], the virtual
// k~, v~, beta~ are the same memory viewed as [B, T n_h, H, d]; only q~ and g~
// are materialised (expand kernel).  On the tensor-core path the state pass
// writes the kept outputs straight into out; the CUDA-core path writes every
// virtual row and a gather kernel keeps every n_h-th.
#include "common.cuh"

namespace gdr_host {
gdr_status fwd_keep(const void *q, const void *k, const void *v, const float *g, const float *beta,
                    const float *S0, void *out, float *S_final, int B, int T, int H, int d_k,
                    int d_v, int chunk, const int32_t *cu_seqlens, int n_seq, gdr_dtype dtype,
                    gdr_gate gate, gdr_path path, void *workspace, size_t workspace_bytes,
                    void *stream, int keep, bool *ran);
}  // namespace gdr_host

namespace gdr {

// Both remap kernels are HBM-bound copies.  A CTA takes whole tokens (the
// virtual rows of one token are contiguous: n_h substeps x H heads), its
// threads stride over 16-byte vectors inside the token, so the only index
// arithmetic is one 32-bit division per vector.  d_k and d_v are multiples of
// 16 elements and rows start 16-byte aligned.  Streaming loads and stores:
// nothing is re-read.

// q~ [ntok * nh, H, dk] and g~ from q [ntok, H, dk] and g [ntok, H(, dk)].
template <typename Tin, bool CH>
__global__ void __launch_bounds__(256) gdp_expand_kernel(const Tin *__restrict__ q,
                                                         const float *__restrict__ g,
                                                         Tin *__restrict__ qv,
                                                         float *__restrict__ gv, long n_tokens,
                                                         int H, int dk, int nh, unsigned int *err) {
    // checked build: the 16-byte vectors tile every row exactly
    if (kChecked && !chk_true((dk * (int)sizeof(Tin)) % 16 == 0 && (!CH || dk % 4 == 0) && nh >= 1, err))
        return;
    const int hq = H * (dk * (int)sizeof(Tin) / 16);  // q vectors of one token
    const int hg = CH ? H * (dk / 4) : H;              // g floats4 (or floats) of one token
    const uint4 *q4 = reinterpret_cast<const uint4 *>(q);
    uint4 *qv4 = reinterpret_cast<uint4 *>(qv);
    for (long t = blockIdx.x; t < n_tokens; t += gridDim.x) {
        const uint4 *src = q4 + t * hq;
        uint4 *dst = qv4 + t * nh * (long)hq;
        for (int w = threadIdx.x; w < nh * hq; w += blockDim.x) {
            const int j = w / hq;  // substep
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (j == nh - 1) val = __ldcs(src + (w - j * hq));
            __stcs(dst + w, val);
        }
        if (CH) {
            const float4 *gs = reinterpret_cast<const float4 *>(g) + t * hg;
            float4 *gd = reinterpret_cast<float4 *>(gv) + t * nh * (long)hg;
            for (int w = threadIdx.x; w < nh * hg; w += blockDim.x)
                __stcs(gd + w, w < hg ? __ldcs(gs + w) : make_float4(0.f, 0.f, 0.f, 0.f));
        } else {
            const float *gs = g + t * hg;
            float *gd = gv + t * nh * (long)hg;
            for (int w = threadIdx.x; w < nh * hg; w += blockDim.x)
                __stcs(gd + w, w < hg ? __ldcs(gs + w) : 0.f);
        }
    }
}

// out [ntok, H, dv] <- the last substep's rows of o~ [ntok * nh, H, dv].
template <typename Tin>
__global__ void __launch_bounds__(256) gdp_gather_kernel(const Tin *__restrict__ ov,
                                                         Tin *__restrict__ out, long n_tokens,
                                                         int H, int dv, int nh, unsigned int *err) {
    if (kChecked && !chk_true((dv * (int)sizeof(Tin)) % 16 == 0 && nh >= 1, err)) return;
    const int ho = H * (dv * (int)sizeof(Tin) / 16);
    const uint4 *ov4 = reinterpret_cast<const uint4 *>(ov);
    uint4 *out4 = reinterpret_cast<uint4 *>(out);
    for (long t = blockIdx.x; t < n_tokens; t += gridDim.x) {
        const uint4 *src = ov4 + (t * nh + nh - 1) * (long)ho;
        uint4 *dst = out4 + t * ho;
        for (int w = threadIdx.x; w < ho; w += blockDim.x) __stcs(dst + w, __ldcs(src + w));
    }
}

__global__ void gdp_scale_offsets_kernel(const int32_t *__restrict__ cu, int32_t *__restrict__ cuv,
                                         int n, int nh, unsigned int *err) {
    if (kChecked && !chk_true(n >= 1 && nh >= 1, err)) return;
    for (int i = threadIdx.x; i <= n; i += blockDim.x) cuv[i] = cu[i] * nh;
}

}  // namespace gdr

using namespace gdr;

namespace {

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

struct GdpLayout {
    size_t qv, gv, ov, cuv, inner, total;
};

GdpLayout gdp_layout(int B, int T, int H, int nh, int dk, int dv, int chunk, int n_seq, int varlen,
                     gdr_dtype dtype, gdr_gate gate, gdr_path path) {
    GdpLayout L;
    const size_t vtok = (size_t)B * T * nh, es = dtype == GDR_BF16 ? 2 : 4;
    size_t o = 0;
    L.qv = o;  o += up256(vtok * H * dk * es);
    L.gv = o;  o += up256(vtok * H * (gate == GDR_GATE_PER_KEY_CHANNEL ? dk : 1) * 4);
    L.ov = o;  o += up256(vtok * H * dv * es);
    L.cuv = o; o += up256((size_t)(varlen ? n_seq + 1 : 1) * 4);
    L.inner = o;
    o += up256(gdr_fwd_workspace_size(B, (int)((long)T * nh), H, dk, dv, chunk, n_seq, varlen,
                                      dtype, gate, path));
    L.total = o;
    return L;
}

bool aligned16(const void *p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }

// Grid of a remap kernel: one CTA per token, at most 8 CTAs of 256 threads
// per SM (148 SMs), the CTAs then loop over tokens.
unsigned copy_grid(long n_tokens) {
    const long cap = 148L * 8;
    return (unsigned)(n_tokens < 1 ? 1 : (n_tokens > cap ? cap : n_tokens));
}

}  // namespace

extern "C" {

size_t gdr_fwd_product_workspace_size(int B, int T, int H, int n_h, int d_k, int d_v, int chunk,
                                      int n_seq, int varlen, gdr_dtype dtype, gdr_gate gate,
                                      gdr_path path) {
    if (B < 1 || T < 0 || H < 1 || n_h < 1 || d_k < 1 || d_v < 1) return 0;
    if ((double)T * n_h > 2.0e9 / (B > 0 ? B : 1)) return 0;
    return gdp_layout(B, T, H, n_h, d_k, d_v, chunk, n_seq, varlen, dtype, gate, path).total;
}

gdr_status gdr_fwd_product(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const float *S0, void *out, float *S_final, int B,
                           int T, int H, int n_h, int d_k, int d_v, int chunk,
                           const int32_t *cu_seqlens, int n_seq, gdr_dtype dtype, gdr_gate gate,
                           gdr_path path, void *workspace, size_t workspace_bytes, void *stream) {
    if (n_h < 1 || B < 1 || T < 0 || H < 1 || d_k < 1 || d_v < 1) return GDR_ERR_INVALID;
    // every path of the gated delta rule takes d_k, d_v multiples of 16 up to 128;
    // checked here too because the remap kernels copy 16-byte row vectors
    if (d_k % 16 || d_v % 16 || d_k > 128 || d_v > 128) return GDR_ERR_UNSUPPORTED;
    if (!(dtype == GDR_F32 || dtype == GDR_BF16) ||
        !(gate == GDR_GATE_SCALAR || gate == GDR_GATE_PER_KEY_CHANNEL))
        return GDR_ERR_INVALID;
    if ((long long)B * T > 0 && (!q || !k || !v || !g || !beta || !out)) return GDR_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(beta) ||
        !aligned16(out) || !aligned16(workspace))
        return GDR_ERR_INVALID;
    if ((double)B * T * n_h > 2.0e9 || (double)B * T * H > 2.0e9) return GDR_ERR_INVALID;
    if ((double)n_h * H * 128 > 2.0e9) return GDR_ERR_INVALID;  // 32-bit per-token vector counts
    const int varlen = cu_seqlens != nullptr;
    if (varlen && (B != 1 || n_seq < 1)) return GDR_ERR_INVALID;
    if (n_h == 1)  // no substeps to flatten: plain gated delta rule
        return gdr_fwd(q, k, v, g, beta, S0, out, S_final, B, T, H, d_k, d_v, chunk, cu_seqlens,
                       n_seq, dtype, gate, path, workspace, workspace_bytes, stream);
    const GdpLayout L = gdp_layout(B, T, H, n_h, d_k, d_v, chunk, n_seq, varlen, dtype, gate, path);
    if (!workspace || workspace_bytes < L.total) return GDR_ERR_INVALID;
    uint8_t *ws = (uint8_t *)workspace;
    void *qv = ws + L.qv, *ov = ws + L.ov;
    float *gv = (float *)(ws + L.gv);
    int32_t *cuv = varlen ? (int32_t *)(ws + L.cuv) : nullptr;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned int *cerr = kChecked ? gdr_host::device_error_word() : nullptr;  // checked build
    const long ntok = (long)B * T;
    const bool ch = gate == GDR_GATE_PER_KEY_CHANNEL;
    if (ntok > 0) {
        const unsigned grid = copy_grid(ntok);
        gdr_host::ProfToken tk = gdr_host::prof_begin(GDR_K_GDP_REMAP, st);
        if (dtype == GDR_BF16) {
            if (ch)
                gdp_expand_kernel<__nv_bfloat16, true><<<grid, 256, 0, st>>>(
                    (const __nv_bfloat16 *)q, g, (__nv_bfloat16 *)qv, gv, ntok, H, d_k, n_h, cerr);
            else
                gdp_expand_kernel<__nv_bfloat16, false><<<grid, 256, 0, st>>>(
                    (const __nv_bfloat16 *)q, g, (__nv_bfloat16 *)qv, gv, ntok, H, d_k, n_h, cerr);
        } else {
            if (ch)
                gdp_expand_kernel<float, true><<<grid, 256, 0, st>>>((const float *)q, g,
                                                                     (float *)qv, gv, ntok, H,
                                                                     d_k, n_h, cerr);
            else
                gdp_expand_kernel<float, false><<<grid, 256, 0, st>>>((const float *)q, g,
                                                                      (float *)qv, gv, ntok, H,
                                                                      d_k, n_h, cerr);
        }
        gdr_host::prof_end(tk, st);
        if (cudaGetLastError() != cudaSuccess) return GDR_ERR_CUDA;
    }
    if (varlen) {
        gdp_scale_offsets_kernel<<<1, 256, 0, st>>>(cu_seqlens, cuv, n_seq, n_h, cerr);
        if (cudaGetLastError() != cudaSuccess) return GDR_ERR_CUDA;
    }
    // the tensor-core path writes the kept rows itself; otherwise gather them
    bool ran = false;
    gdr_status s = gdr_host::fwd_keep(qv, k, v, gv, beta, S0, out, S_final, B,
                                      (int)((long)T * n_h), H, d_k, d_v, chunk, cuv, n_seq, dtype,
                                      gate, path, ws + L.inner, workspace_bytes - L.inner, stream,
                                      n_h, &ran);
    if (s != GDR_OK || ran) return s;
    s = gdr_fwd(qv, k, v, gv, beta, S0, ov, S_final, B, (int)((long)T * n_h), H, d_k, d_v, chunk,
                cuv, n_seq, dtype, gate, path, ws + L.inner, workspace_bytes - L.inner, stream);
    if (s != GDR_OK) return s;
    if (ntok > 0) {
        const unsigned grid = copy_grid(ntok);
        gdr_host::ProfToken tk = gdr_host::prof_begin(GDR_K_GDP_REMAP, st);
        if (dtype == GDR_BF16)
            gdp_gather_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
                (const __nv_bfloat16 *)ov, (__nv_bfloat16 *)out, ntok, H, d_v, n_h, cerr);
        else
            gdp_gather_kernel<float><<<grid, 256, 0, st>>>((const float *)ov, (float *)out, ntok,
                                                           H, d_v, n_h, cerr);
        gdr_host::prof_end(tk, st);
        if (cudaGetLastError() != cudaSuccess) return GDR_ERR_CUDA;
    }
    return GDR_OK;
}

}  // extern "C"
