// C-ABI entry points of libgdr: host-side validation, workspace sizing and
// dispatch to the kernels.  Declared in include/gdr.h.
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "sm100.cuh"

namespace gdr_host {
cudaError_t decode_dispatch(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float *S, void *out, int N, int H, int dk, int dv,
                            gdr_dtype dtype, gdr_gate gate, cudaStream_t st);
cudaError_t fwd_simt_dispatch(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *S0, void *out, float *S_final,
                              int T, int H, int dk, int dv, int C, const int32_t *cu, int n_seq,
                              int T_total, gdr_dtype dtype, gdr_gate gate, cudaStream_t st);
size_t simt_smem_bytes(int C, int dk, bool channel, bool dec);
cudaError_t fwd_simt_gdn2_dispatch(const void *q, const void *k, const void *v, const float *g,
                                   const float *eg, const float *wg, const float *S0, void *out,
                                   float *S_final, int T, int H, int dk, int dv, int C,
                                   const int32_t *cu, int n_seq, int T_total, gdr_dtype dtype,
                                   gdr_gate gate, cudaStream_t st);
cudaError_t fwd_tc_gdn2_dispatch(const void *q, const void *k, const void *v, const float *g,
                                 const float *eg, const float *wg, const float *S0, void *out,
                                 float *S_final, int B, int T, int H, const int32_t *cu, int n_seq,
                                 gdr_gate gate, void *workspace, size_t ws_bytes,
                                 unsigned int *err, cudaStream_t st, int chunk);
size_t tc_workspace_bytes_gdn2_chunk(int B, int T, int H, int n_seq, int varlen, int chunk);
cudaError_t decode_gdn2_dispatch(const void *q, const void *k, const void *v, const float *g,
                                 const float *eg, const float *wg, float *S, void *out, int N,
                                 int H, int dk, int dv, gdr_dtype dtype, gdr_gate gate,
                                 cudaStream_t st);
// tensor-core path (fwd_tc.cu)
bool tc_applies(int dk, int dv, int chunk, gdr_dtype dtype);
bool tc_applies_fwd(int dk, int dv, int chunk, gdr_dtype dtype, gdr_gate gate, int keep);
size_t tc_workspace_bytes(int B, int T, int H, int n_seq, int varlen, gdr_gate gate);
size_t tc_workspace_bytes_chunk(int B, int T, int H, int n_seq, int varlen, gdr_gate gate,
                                int chunk);
cudaError_t fwd_tc_dispatch(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *S0, void *out, float *S_final, int B,
                            int T, int H, const int32_t *cu, int n_seq, gdr_gate gate,
                            void *workspace, size_t ws_bytes, unsigned int *err, cudaStream_t st,
                            int chunk);
cudaError_t fwd_tc_keep_dispatch(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *S0, void *out, float *S_final,
                                 int B, int T, int H, const int32_t *cu, int n_seq, gdr_gate gate,
                                 int keep, void *workspace, size_t ws_bytes, unsigned int *err,
                                 cudaStream_t st, int chunk);
}  // namespace gdr_host

// ------------------------------------------------------------ device error word
static __device__ unsigned int g_gdr_device_error;

namespace gdr_host {
// Cached per device; entries are atomic because host threads may make their
// first call on a device at the same time (both store the same address).
unsigned int *device_error_word() {
    static std::atomic<unsigned int *> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    unsigned int *w = cache[dev].load(std::memory_order_acquire);
    if (!w) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_gdr_device_error) != cudaSuccess) return nullptr;
        w = (unsigned int *)p;
        cache[dev].store(w, std::memory_order_release);
    }
    return w;
}
}  // namespace gdr_host

// ------------------------------------------------------------ launch accounting
namespace {
struct ProfPending {
    int id;
    cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::atomic<long long> g_launches[GDR_K_COUNT];
long long g_launch_base[GDR_K_COUNT];
double g_prof_ms[GDR_K_COUNT];
std::vector<ProfPending> g_pending;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}
}  // namespace

namespace gdr_host {
ProfToken prof_begin(int id, cudaStream_t st) {
    g_launches[id].fetch_add(1);
    ProfToken t{id, -1};
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof_on) return t;
    cudaEvent_t a = take_event(), b = take_event();
    if (!a || !b) return t;
    cudaEventRecord(a, st);
    g_pending.push_back({id, a, b});
    t.slot = (int)g_pending.size() - 1;
    return t;
}
void prof_end(ProfToken tok, cudaStream_t st) {
    if (tok.slot < 0) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (tok.slot < (int)g_pending.size()) cudaEventRecord(g_pending[tok.slot].b, st);
}
}  // namespace gdr_host

namespace {

bool aligned16(const void *p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }

bool valid_enum(gdr_dtype d, gdr_gate g) {
    return (d == GDR_F32 || d == GDR_BF16) && (g == GDR_GATE_SCALAR || g == GDR_GATE_PER_KEY_CHANNEL);
}

bool simt_shape_ok(int dk, int dv, int chunk) {
    return dk >= 16 && dk <= 128 && dk % 16 == 0 && dv >= 16 && dv <= 128 && dv % 16 == 0 &&
           (chunk == 16 || chunk == 32 || chunk == 64 || chunk == 128);
}

// Resolve the path; returns GDR_OK and sets *use_tc, or an error.
gdr_status resolve_path(int dk, int dv, int chunk, gdr_dtype dtype, gdr_gate gate, int keep,
                        gdr_path path, bool *use_tc) {
    const bool tc = gdr_host::tc_applies_fwd(dk, dv, chunk, dtype, gate, keep);
    switch (path) {
        case GDR_PATH_AUTO:
            *use_tc = tc;
            break;
        case GDR_PATH_SIMT:
            *use_tc = false;
            break;
        case GDR_PATH_TENSORCORE:
            if (!tc) return GDR_ERR_UNSUPPORTED;
            *use_tc = true;
            break;
        default:
            return GDR_ERR_INVALID;
    }
    if (!*use_tc && !simt_shape_ok(dk, dv, chunk)) return GDR_ERR_UNSUPPORTED;
    return GDR_OK;
}

// Gated DeltaNet-2 takes the tensor-core path with either decay.
gdr_status resolve_gdn2_path(int dk, int dv, int chunk, gdr_dtype dtype, gdr_gate gate,
                             gdr_path path, bool *use_tc) {
    const bool tc = gdr_host::tc_applies_fwd(dk, dv, chunk, dtype, gate, 1);
    switch (path) {
        case GDR_PATH_AUTO: *use_tc = tc; break;
        case GDR_PATH_SIMT: *use_tc = false; break;
        case GDR_PATH_TENSORCORE:
            if (!tc) return GDR_ERR_UNSUPPORTED;
            *use_tc = true;
            break;
        default: return GDR_ERR_INVALID;
    }
    if (!*use_tc && !simt_shape_ok(dk, dv, chunk)) return GDR_ERR_UNSUPPORTED;
    return GDR_OK;
}

gdr_status check_fwd_shapes(int B, int T, int H, int dk, int dv, int chunk, int n_seq, bool varlen) {
    if (B < 1 || T < 0 || H < 1 || dk < 1 || dv < 1) return GDR_ERR_INVALID;
    if (chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return GDR_ERR_INVALID;
    if (varlen && (B != 1 || n_seq < 1)) return GDR_ERR_INVALID;
    // element counts must stay addressable with 64-bit offsets and 32-bit grid/TMA coordinates
    const double tokens = (double)B * (double)T;
    if (tokens * H * (dk > dv ? dk : dv) > 9.0e15 || tokens > 2.0e9) return GDR_ERR_INVALID;
    if ((double)(varlen ? n_seq : B) * H > 2.0e9) return GDR_ERR_INVALID;
    return GDR_OK;
}

}  // namespace

extern "C" {

const char *gdr_status_string(gdr_status s) {
    switch (s) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_INVALID: return "GDR_ERR_INVALID: invalid argument";
        case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED: sizes or path not built";
        case GDR_ERR_CUDA: return "GDR_ERR_CUDA: CUDA runtime error";
        case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT: a bounded device wait expired";
        case GDR_ERR_BOUNDS: return "GDR_ERR_BOUNDS: a bounds guard refused an access";
    }
    return "GDR_ERR_UNKNOWN";
}

size_t gdr_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int chunk, int n_seq,
                              int varlen, gdr_dtype dtype, gdr_gate gate, gdr_path path) {
    if (!valid_enum(dtype, gate)) return 0;
    if (check_fwd_shapes(B, T, H, d_k, d_v, chunk, n_seq, varlen != 0) != GDR_OK) return 0;
    bool use_tc = false;
    if (resolve_path(d_k, d_v, chunk, dtype, gate, 1, path, &use_tc) != GDR_OK) return 0;
    if (!use_tc) return 0;
    return gdr_host::tc_workspace_bytes_chunk(B, T, H, n_seq, varlen, gate, chunk);
}

// The prefill behind gdr_fwd.  keep > 1 (Gated DeltaProduct): the T rows of a
// sequence are keep substeps per token and out holds one row per token, the
// last substep's; only the tensor-core path does this, and where it does not
// apply *ran is false and nothing is launched.
static gdr_status fwd_common(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *S0, void *out, float *S_final, int B,
                             int T, int H, int d_k, int d_v, int chunk,
                             const int32_t *cu_seqlens, int n_seq, gdr_dtype dtype, gdr_gate gate,
                             gdr_path path, void *workspace, size_t workspace_bytes, void *stream,
                             int keep, bool *ran) {
    if (ran) *ran = false;
    // With no tokens (B*T == 0) the token tensors are empty and may be NULL.
    if ((long long)B * T > 0 && (!q || !k || !v || !g || !beta || !out)) return GDR_ERR_INVALID;
    if (!valid_enum(dtype, gate)) return GDR_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(beta) ||
        !aligned16(S0) || !aligned16(out) || !aligned16(S_final) || !aligned16(cu_seqlens))
        return GDR_ERR_INVALID;
    const bool varlen = cu_seqlens != nullptr;
    gdr_status st = check_fwd_shapes(B, T, H, d_k, d_v, chunk, n_seq, varlen);
    if (st != GDR_OK) return st;
    bool use_tc = false;
    st = resolve_path(d_k, d_v, chunk, dtype, gate, keep, path, &use_tc);
    if (st != GDR_OK) return st;
    if (keep > 1 && (!use_tc || T % keep)) return GDR_OK;  // the caller gathers
    if (ran) *ran = true;
    const int nseq = varlen ? n_seq : B;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (use_tc) {  // the dispatcher accounts for its own launches
        const size_t need = gdr_host::tc_workspace_bytes_chunk(B, T, H, n_seq, varlen, gate, chunk);
        if (need && (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u)))
            return GDR_ERR_INVALID;
        e = keep > 1 ? gdr_host::fwd_tc_keep_dispatch(q, k, v, g, beta, S0, out, S_final, B, T, H,
                                                      cu_seqlens, nseq, gate, keep, workspace,
                                                      workspace_bytes,
                                                      gdr_host::device_error_word(), s, chunk)
                     : gdr_host::fwd_tc_dispatch(q, k, v, g, beta, S0, out, S_final, B, T, H,
                                                 cu_seqlens, nseq, gate, workspace,
                                                 workspace_bytes, gdr_host::device_error_word(), s,
                                                 chunk);
    } else {
        if ((size_t)gdr_host::simt_smem_bytes(chunk, d_k, gate == GDR_GATE_PER_KEY_CHANNEL,
                                              false) > 227u * 1024u)
            return GDR_ERR_UNSUPPORTED;
        gdr_host::ProfToken tk = gdr_host::prof_begin(GDR_K_FWD_SIMT, s);
        e = gdr_host::fwd_simt_dispatch(q, k, v, g, beta, S0, out, S_final, T, H, d_k, d_v, chunk,
                                        cu_seqlens, nseq, B * T, dtype, gate, s);
        gdr_host::prof_end(tk, s);
    }
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

gdr_status gdr_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                   const float *S0, void *out, float *S_final, int B, int T, int H, int d_k,
                   int d_v, int chunk, const int32_t *cu_seqlens, int n_seq, gdr_dtype dtype,
                   gdr_gate gate, gdr_path path, void *workspace, size_t workspace_bytes,
                   void *stream) {
    return fwd_common(q, k, v, g, beta, S0, out, S_final, B, T, H, d_k, d_v, chunk, cu_seqlens,
                      n_seq, dtype, gate, path, workspace, workspace_bytes, stream, 1, nullptr);
}

gdr_status gdr_decode_step(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, float *S_inout, void *out, int N, int H, int d_k,
                           int d_v, gdr_dtype dtype, gdr_gate gate, void *stream) {
    if (!q || !k || !v || !g || !beta || !S_inout || !out) return GDR_ERR_INVALID;
    if (!valid_enum(dtype, gate)) return GDR_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(beta) ||
        !aligned16(S_inout) || !aligned16(out))
        return GDR_ERR_INVALID;
    if (N < 1 || H < 1 || d_k < 1 || d_v < 1) return GDR_ERR_INVALID;
    if ((double)N * H > 2.0e9) return GDR_ERR_INVALID;
    if (!(d_k == 64 || d_k == 128) || d_v % 32 != 0 || d_v > 256) return GDR_ERR_UNSUPPORTED;
    gdr_host::ProfToken tk = gdr_host::prof_begin(GDR_K_DECODE, (cudaStream_t)stream);
    cudaError_t e = gdr_host::decode_dispatch(q, k, v, g, beta, S_inout, out, N, H, d_k, d_v,
                                              dtype, gate, (cudaStream_t)stream);
    gdr_host::prof_end(tk, (cudaStream_t)stream);
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

size_t gdr_fwd_gdn2_workspace_size(int B, int T, int H, int d_k, int d_v, int chunk, int n_seq,
                                   int varlen, gdr_dtype dtype, gdr_gate gate, gdr_path path) {
    if (!valid_enum(dtype, gate)) return 0;
    if (check_fwd_shapes(B, T, H, d_k, d_v, chunk, n_seq, varlen != 0) != GDR_OK) return 0;
    bool use_tc = false;
    if (resolve_gdn2_path(d_k, d_v, chunk, dtype, gate, path, &use_tc) != GDR_OK) return 0;
    if (!use_tc) return 0;
    return gdr_host::tc_workspace_bytes_gdn2_chunk(B, T, H, n_seq, varlen, chunk);
}

gdr_status gdr_fwd_gdn2(const void *q, const void *k, const void *v, const float *g,
                        const float *b, const float *w, const float *S0, void *out,
                        float *S_final, int B, int T, int H, int d_k, int d_v, int chunk,
                        const int32_t *cu_seqlens, int n_seq, gdr_dtype dtype, gdr_gate gate,
                        gdr_path path, void *workspace, size_t workspace_bytes, void *stream) {
    if ((long long)B * T > 0 && (!q || !k || !v || !g || !b || !w || !out)) return GDR_ERR_INVALID;
    if (!valid_enum(dtype, gate)) return GDR_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(b) ||
        !aligned16(w) || !aligned16(S0) || !aligned16(out) || !aligned16(S_final) ||
        !aligned16(cu_seqlens))
        return GDR_ERR_INVALID;
    const bool varlen = cu_seqlens != nullptr;
    gdr_status st = check_fwd_shapes(B, T, H, d_k, d_v, chunk, n_seq, varlen);
    if (st != GDR_OK) return st;
    bool use_tc = false;
    st = resolve_gdn2_path(d_k, d_v, chunk, dtype, gate, path, &use_tc);
    if (st != GDR_OK) return st;
    const int nseq = varlen ? n_seq : B;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (use_tc) {  // the dispatcher accounts for its own launches
        const size_t need = gdr_host::tc_workspace_bytes_gdn2_chunk(B, T, H, n_seq, varlen, chunk);
        if (need && (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u)))
            return GDR_ERR_INVALID;
        e = gdr_host::fwd_tc_gdn2_dispatch(q, k, v, g, b, w, S0, out, S_final, B, T, H,
                                           cu_seqlens, nseq, gate, workspace, workspace_bytes,
                                           gdr_host::device_error_word(), s, chunk);
    } else {
        if (gdr_host::simt_smem_bytes(chunk, d_k, gate == GDR_GATE_PER_KEY_CHANNEL, true) >
            227u * 1024u)
            return GDR_ERR_UNSUPPORTED;
        gdr_host::ProfToken tk = gdr_host::prof_begin(GDR_K_GDN2_SIMT, s);
        e = gdr_host::fwd_simt_gdn2_dispatch(q, k, v, g, b, w, S0, out, S_final, T, H, d_k, d_v,
                                             chunk, cu_seqlens, nseq, B * T, dtype, gate, s);
        gdr_host::prof_end(tk, s);
    }
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

gdr_status gdr_decode_step_gdn2(const void *q, const void *k, const void *v, const float *g,
                                const float *b, const float *w, float *S_inout, void *out, int N,
                                int H, int d_k, int d_v, gdr_dtype dtype, gdr_gate gate,
                                void *stream) {
    if (!q || !k || !v || !g || !b || !w || !S_inout || !out) return GDR_ERR_INVALID;
    if (!valid_enum(dtype, gate)) return GDR_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(b) ||
        !aligned16(w) || !aligned16(S_inout) || !aligned16(out))
        return GDR_ERR_INVALID;
    if (N < 1 || H < 1 || d_k < 1 || d_v < 1) return GDR_ERR_INVALID;
    if ((double)N * H > 2.0e9) return GDR_ERR_INVALID;
    if (!(d_k == 64 || d_k == 128) || d_v % 32 != 0 || d_v > 256) return GDR_ERR_UNSUPPORTED;
    gdr_host::ProfToken tk = gdr_host::prof_begin(GDR_K_GDN2_DECODE, (cudaStream_t)stream);
    cudaError_t e = gdr_host::decode_gdn2_dispatch(q, k, v, g, b, w, S_inout, out, N, H, d_k, d_v,
                                                   dtype, gate, (cudaStream_t)stream);
    gdr_host::prof_end(tk, (cudaStream_t)stream);
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // extern "C"

namespace gdr_host {
// Gated DeltaProduct over its virtual sequence (T = n_h x tokens rows per
// sequence), writing only the last substep of each token into out; *ran is
// false where the tensor-core path does not apply and nothing was launched.
gdr_status fwd_keep(const void *q, const void *k, const void *v, const float *g, const float *beta,
                    const float *S0, void *out, float *S_final, int B, int T, int H, int d_k,
                    int d_v, int chunk, const int32_t *cu_seqlens, int n_seq, gdr_dtype dtype,
                    gdr_gate gate, gdr_path path, void *workspace, size_t workspace_bytes,
                    void *stream, int keep, bool *ran) {
    return fwd_common(q, k, v, g, beta, S0, out, S_final, B, T, H, d_k, d_v, chunk, cu_seqlens,
                      n_seq, dtype, gate, path, workspace, workspace_bytes, stream, keep, ran);
}
}  // namespace gdr_host

// ------------------------------------------------------------ error-path self test
static __global__ void wait_timeout_kernel(unsigned int spin_limit, unsigned int *err) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        gdr::sm100::mbar_init(&bar, 1);
        gdr::sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // Nobody arrives: phase 0 never completes, the bounded wait gives up.
        gdr::sm100::mbar_wait_bounded(&bar, 0, spin_limit, err);
    }
}

// A guarded write one element past a 16-float array: the guard refuses it.
static __device__ float g_bounds_scratch[16];
static __global__ void bounds_selftest_kernel(float *scratch, unsigned int *err) {
    const long long i = 16 + threadIdx.x;
    if (gdr::chk_span(i, 1, 16, err)) scratch[i] = 1.f;
}

extern "C" {

int gdr_checked_build(void) { return gdr::kChecked ? 1 : 0; }

gdr_status gdr_selftest_bounds(void *stream) {
    if (!gdr::kChecked) return GDR_ERR_UNSUPPORTED;
    unsigned int *err = gdr_host::device_error_word();
    if (!err) return GDR_ERR_CUDA;
    float *p = nullptr;
    if (cudaGetSymbolAddress((void **)&p, g_bounds_scratch) != cudaSuccess) return GDR_ERR_CUDA;
    bounds_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(p, err);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

gdr_status gdr_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return GDR_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_gdr_device_error, sizeof(word)) != cudaSuccess)
        return GDR_ERR_CUDA;
    if (word && cudaMemcpyToSymbol(g_gdr_device_error, &zero, sizeof(zero)) != cudaSuccess)
        return GDR_ERR_CUDA;
    if (word & gdr::kErrTimeout) return GDR_ERR_TIMEOUT;
    if (word & gdr::kErrBounds) return GDR_ERR_BOUNDS;
    return (word & gdr::kErrNumeric) ? GDR_ERR_INVALID : GDR_OK;
}

void gdr_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = on != 0;
}

gdr_status gdr_profile_read(int id, long long *launches, double *total_ms) {
    if (id < 0 || id >= GDR_K_COUNT) return GDR_ERR_INVALID;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    gdr_status st = GDR_OK;
    std::vector<ProfPending> keep;
    for (auto &p : g_pending) {
        if (cudaEventSynchronize(p.b) != cudaSuccess) st = GDR_ERR_CUDA;
        float ms = 0.f;
        if (st == GDR_OK && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess)
            g_prof_ms[p.id] += ms;
        g_event_pool.push_back(p.a);
        g_event_pool.push_back(p.b);
    }
    g_pending.clear();
    const long long now = g_launches[id].load();
    if (launches) *launches = now - g_launch_base[id];
    if (total_ms) *total_ms = g_prof_ms[id];
    g_launch_base[id] = now;
    g_prof_ms[id] = 0.0;
    return st;
}

gdr_status gdr_selftest_wait_timeout(unsigned int spin_limit, void *stream) {
    if (spin_limit == 0 || spin_limit > (1u << 24)) return GDR_ERR_INVALID;
    unsigned int *err = gdr_host::device_error_word();
    if (!err) return GDR_ERR_CUDA;
    wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(spin_limit, err);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // extern "C"
