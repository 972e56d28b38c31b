// gdr_fwd_noalloc: the tensor-core prefill with its scratch memory taken from
// a fixed array inside this library instead of from the caller.
//
// Who needs it: callers that may not allocate device memory at call time --
// e.g. a host program whose memory manager reserves the whole device heap up
// front and forbids any further cudaMalloc, or a latency-critical loop where
// an allocation (which can synchronise the device) is not acceptable -- and
// that also cannot hand the library a workspace of their own.
//
// The scratch is one file-scope device array of kNoAllocScratchBytes bytes.
// Every device that loads this library holds it until the process exits.
#include <atomic>

#include "common.cuh"

namespace gdr_host {
bool tc_applies(int dk, int dv, int chunk, gdr_dtype dtype);
size_t tc_workspace_bytes(int B, int T, int H, int n_seq, int varlen, gdr_gate gate);
cudaError_t fwd_tc_dispatch(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *S0, void *out, float *S_final, int B,
                            int T, int H, const int32_t *cu, int n_seq, gdr_gate gate,
                            void *workspace, size_t ws_bytes, unsigned int *err, cudaStream_t st,
                            int chunk);
}  // namespace gdr_host

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;  // 32 MiB

// The shared scratch.  In host code this name is only a stand-in for the
// device symbol: its device address comes from cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch on the current device, looked up once per
// device (the first gdr_fwd_noalloc call on that device does the lookup).
// Host threads may race on a device's first call: each entry is atomic, and
// two concurrent lookups store the same address.
void *scratch_address(int *status) {
    static std::atomic<void *> addr[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        *status = GDR_ERR_CUDA;
        return nullptr;
    }
    void *p = addr[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            *status = GDR_ERR_CUDA;
            return nullptr;
        }
        addr[dev].store(p, std::memory_order_release);
    }
    *status = GDR_OK;
    return p;
}

bool aligned16(const void *p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" {

size_t gdr_fwd_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

gdr_status gdr_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const float *S0, void *out, float *S_final, int B,
                           int T, int H, int d_k, int d_v, int chunk, const int32_t *cu_seqlens,
                           int n_seq, gdr_dtype dtype, gdr_gate gate, void *stream) {
    if ((long long)B * T > 0 && (!q || !k || !v || !g || !beta || !out)) return GDR_ERR_INVALID;
    if (!(dtype == GDR_F32 || dtype == GDR_BF16) ||
        !(gate == GDR_GATE_SCALAR || gate == GDR_GATE_PER_KEY_CHANNEL))
        return GDR_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(beta) ||
        !aligned16(S0) || !aligned16(out) || !aligned16(S_final) || !aligned16(cu_seqlens))
        return GDR_ERR_INVALID;
    if (B < 1 || T < 0 || H < 1) return GDR_ERR_INVALID;
    const bool varlen = cu_seqlens != nullptr;
    if (varlen && (B != 1 || n_seq < 1)) return GDR_ERR_INVALID;
    if ((double)B * T > 2.0e9 || (double)(varlen ? n_seq : B) * H > 2.0e9) return GDR_ERR_INVALID;
    if (!gdr_host::tc_applies(d_k, d_v, chunk, dtype)) return GDR_ERR_UNSUPPORTED;
    const size_t need = gdr_host::tc_workspace_bytes(B, T, H, n_seq, varlen, gate);
    if (need > kNoAllocScratchBytes) return GDR_ERR_UNSUPPORTED;  // larger than the fixed scratch
    int st = GDR_OK;
    void *scratch = scratch_address(&st);
    if (!scratch) return (gdr_status)st;
    // Nothing in the scratch has to start at zero: every tile a kernel reads
    // was written earlier in the same call.
    cudaError_t e = gdr_host::fwd_tc_dispatch(q, k, v, g, beta, S0, out, S_final, B, T, H,
                                              cu_seqlens, varlen ? n_seq : B, gate, scratch,
                                              kNoAllocScratchBytes, gdr_host::device_error_word(),
                                              (cudaStream_t)stream, 64);
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // extern "C"
