/*
 * gdr.h -- C-ABI of the B200 (sm_100a) gated delta rule forward pass.
 *
 * The operation (column convention; the state S of one (sequence, head) is a
 * d_v x d_k fp32 matrix, q_t, k_t in R^{d_k}, v_t in R^{d_v}):
 *
 *     S_t = (S_{t-1} D_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,    o_t = S_t q_t
 *
 * with D_t = exp(g_t) I  (GDR_GATE_SCALAR, Gated DeltaNet) or
 *      D_t = Diag(exp(g_t)) (GDR_GATE_PER_KEY_CHANNEL, Kimi Delta Attention:
 *      the state is decayed channel by channel first, then corrected).
 * Sources: "Gated DeltaNet: Householder Transitions and the Arithmetic of
 * Forgetting", section "The gated delta rule"; "Linear Attention, Visualized",
 * sections "Gated DeltaNet (GDN)" and "Kimi Delta Attention (KDA)".
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or keeps them.  Tensors are dense row-major
 *    (contiguous) and 16-byte aligned.
 *  - q, k, v and out are fp32 (GDR_F32) or bf16 (GDR_BF16) as `dtype` says;
 *    g, beta and all states are fp32.
 *  - g is the log of the decay: alpha = exp(g) (g <= 0 for a decay).  beta is
 *    used as given (no clamp; beta = 2 makes the reflection I - 2 k k^T).
 *    No 1/sqrt(d) scale and no normalisation is applied: q and k are used as
 *    given ("Linear Attention, Visualized", Notation: the scale is absorbed
 *    into q or k).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Argument validation happens on the host before any launch; a
 *    failed validation launches nothing and leaves every output untouched.
 *  - `out` must not overlap any input.  S0 may equal S_final (in-place
 *    continuation); other overlaps are not allowed.
 */
#ifndef GDR_H
#define GDR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID = 1,      /* bad shape, NULL where required, misalignment, bad enum */
    GDR_ERR_UNSUPPORTED = 2,  /* valid but not built: sizes or path outside the instantiated set */
    GDR_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    GDR_ERR_TIMEOUT = 4,      /* a bounded device-side wait expired (see gdr_device_status) */
    GDR_ERR_BOUNDS = 5        /* checked build only: a kernel's bounds guard refused an access */
} gdr_status;

typedef enum { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

typedef enum { GDR_GATE_SCALAR = 0, GDR_GATE_PER_KEY_CHANNEL = 1 } gdr_gate;

/* Which kernels run the prefill.
 *  GDR_PATH_AUTO        tensor-core path when it applies (bf16, d_k = d_v = 128,
 *                       chunk = 64 or 16), else the SIMT path.
 *  GDR_PATH_SIMT        fp32 CUDA-core kernels (any supported shape; the only
 *                       path for fp32 inputs).
 *  GDR_PATH_TENSORCORE  tcgen05/TMEM + TMA kernels; GDR_ERR_UNSUPPORTED where
 *                       they do not apply. */
typedef enum { GDR_PATH_AUTO = 0, GDR_PATH_SIMT = 1, GDR_PATH_TENSORCORE = 2 } gdr_path;

/* Human-readable name of a status code (static storage; never NULL). */
const char *gdr_status_string(gdr_status s);

/*
 * Bytes of device workspace gdr_fwd needs for these arguments and this path
 * (0 if none).  Returns 0 as well for arguments gdr_fwd would reject.
 * `n_seq` is the number of packed sequences when cu_seqlens is used, else
 * ignored (pass 0).
 */
size_t gdr_fwd_workspace_size(int B, int T, int H, int d_k, int d_v, int chunk, int n_seq,
                              int varlen, gdr_dtype dtype, gdr_gate gate, gdr_path path);

/*
 * Chunkwise-parallel prefill over whole sequences (the chunked WY/UT form of
 * "Linear Attention, Visualized", sections "Gated DeltaNet (GDN) / Complete
 * per-chunk algorithm" and "Kimi Delta Attention (KDA) / Complete per-chunk
 * algorithm"; the result equals the token recurrence above for every chunk
 * size, section "Chunkwise algorithm / Cost").
 *
 *  q, k     [B, T, H, d_k]   dtype
 *  v        [B, T, H, d_v]   dtype
 *  g        [B, T, H] (GDR_GATE_SCALAR) or [B, T, H, d_k] (per channel), fp32
 *  beta     [B, T, H]        fp32
 *  S0       [N, H, d_v, d_k] fp32 initial states, or NULL for zero states
 *  out      [B, T, H, d_v]   dtype, written for every token
 *           (with B*T == 0 the token tensors may be NULL; S_final = S0)
 *  S_final  [N, H, d_v, d_k] fp32 final states, or NULL to skip
 *  chunk    16, 32, 64 or 128 (SIMT); 64 or 16 (tensor-core path; at 16 a
 *           64-token tile holds four 16-token chunks,
 *           with block-diagonal L, A and T and four chain steps per tile).
 *           Every chunk size gives the token recurrence's result up to
 *           rounding.  At 128 the SIMT path streams the chunk's key channels
 *           through shared memory in blocks of 16 (one CTA per SM); smaller
 *           chunks keep whole tiles resident.
 *  cu_seqlens  NULL: N = B sequences of length T.  Otherwise a DEVICE int32
 *           array [n_seq + 1] of token offsets into a packed batch (B must be
 *           1, cu_seqlens[0] = 0, cu_seqlens[n_seq] = T, non-decreasing); the
 *           state restarts from S0[i] (or zero) at every sequence start and
 *           N = n_seq.  Offsets live on the device and are not read by the
 *           host; out-of-range or decreasing offsets are clamped into [0, T] by
 *           the kernels (never an out-of-bounds access; such results are
 *           unspecified).
 *  d_k, d_v multiples of 16 in [16, 128] (SIMT); 128 (tensor-core path).
 *  workspace / workspace_bytes: device scratch of at least
 *           gdr_fwd_workspace_size(...) bytes, 256-byte aligned, owned by the
 *           caller, not used by anything else until the call has completed on
 *           `stream`.  May be NULL when that size is 0.
 * Returns GDR_OK once the work is enqueued.
 */
gdr_status gdr_fwd(const void *q, const void *k, const void *v, const float *g,
                   const float *beta, const float *S0, void *out, float *S_final, int B, int T,
                   int H, int d_k, int d_v, int chunk, const int32_t *cu_seqlens, int n_seq,
                   gdr_dtype dtype, gdr_gate gate, gdr_path path, void *workspace,
                   size_t workspace_bytes, void *stream);

/*
 * One decode step for N independent sequences, updating the states in place
 * (the token recurrence above applied once; "Linear Attention, Visualized",
 * DeltaNet / Recurrent form, with the decay of section "Gated DeltaNet (GDN)"
 * or "Kimi Delta Attention (KDA)").
 *
 *  q, k     [N, H, d_k]        dtype
 *  v        [N, H, d_v]        dtype
 *  g        [N, H] or [N, H, d_k]  fp32 log-decay
 *  beta     [N, H]             fp32
 *  S_inout  [N, H, d_v, d_k]   fp32, read and overwritten
 *  out      [N, H, d_v]        dtype
 *  d_k in {64, 128}; d_v a multiple of 32 in [32, 256].
 */
gdr_status gdr_decode_step(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, float *S_inout, void *out, int N, int H, int d_k,
                           int d_v, gdr_dtype dtype, gdr_gate gate, void *stream);

/*
 * Synchronises `stream`, then reports (and clears) the device-side error word
 * of the current device: GDR_ERR_TIMEOUT if a bounded wait inside a kernel
 * gave up since the last call (that kernel skipped its remaining work and
 * returned), GDR_ERR_BOUNDS if a guard of the checked build refused an access,
 * GDR_ERR_INVALID if a frame factorisation met a non-positive pivot,
 * GDR_ERR_CUDA if the stream reports an error, else GDR_OK.
 */
gdr_status gdr_device_status(void *stream);

/*
 * Self-test of the bounded-wait error path: launches one tiny kernel that
 * waits on a shared-memory barrier nobody arrives at, gives up after
 * about `spin_limit` polls, records GDR_ERR_TIMEOUT in the device error word and
 * returns normally (the context stays usable).  Follow with gdr_device_status.
 */
gdr_status gdr_selftest_wait_timeout(unsigned int spin_limit, void *stream);

/*
 * The checked build (compiled with -DGDR_CHECK; libgdr_check.so beside
 * libgdr.so): every kernel checks the spans of the global buffers its CTA reads
 * and writes, and its TMA coordinates (x >= 0 and 16-byte aligned, box origin
 * inside the tensor), against the extents of the call before it touches
 * memory.  A failed check sets a bit in the device error word, the CTA returns
 * without touching anything, and gdr_device_status reports GDR_ERR_BOUNDS.
 * The checks cost a few instructions per CTA; results are bit-identical to the
 * normal build's.
 *
 * gdr_checked_build: 1 in the checked build, 0 in the normal one.
 * gdr_selftest_bounds: checked build only (else GDR_ERR_UNSUPPORTED): launches
 * one tiny kernel whose guard refuses an access past the end of a 16-float
 * scratch array (the access is never made), so that the following
 * gdr_device_status reports GDR_ERR_BOUNDS; the context stays usable.
 */
int gdr_checked_build(void);
gdr_status gdr_selftest_bounds(void *stream);

/*
 * Gated DeltaProduct prefill ("Linear Attention, Visualized", section "Gated
 * Delta Product (GDP)"): every token t applies n_h substeps
 *     S <- S (I - beta_tj k_tj k_tj^T) + beta_tj v_tj k_tj^T,   j = 1..n_h,
 * after the token's single decay D_t, and o_t = S q_t is read after the last
 * substep.  Computed, as the page's section "GDP as GDN over a virtual
 * sequence" shows, by the gated delta rule over the n_h T virtual steps with
 * the decay on the first substep and the query on the last; the prefill kernels
 * run unchanged.
 *
 *  q        [B, T, H, d_k]          dtype
 *  k        [B, T, n_h, H, d_k]     dtype (substeps of a token adjacent)
 *  v        [B, T, n_h, H, d_v]     dtype
 *  g        [B, T, H] or [B, T, H, d_k]  fp32 log-decay, one per token
 *  beta     [B, T, n_h, H]          fp32
 *  S0, S_final, out, cu_seqlens (token offsets of real tokens), chunk, path:
 *           as for gdr_fwd.
 *  workspace: at least gdr_fwd_product_workspace_size(...) bytes (holds the
 *           virtual queries and gates, the virtual outputs and the inner
 *           prefill's workspace).  n_h = 1 is gdr_fwd.
 */
size_t gdr_fwd_product_workspace_size(int B, int T, int H, int n_h, int d_k, int d_v, int chunk,
                                      int n_seq, int varlen, gdr_dtype dtype, gdr_gate gate,
                                      gdr_path path);
gdr_status gdr_fwd_product(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const float *S0, void *out, float *S_final, int B,
                           int T, int H, int n_h, int d_k, int d_v, int chunk,
                           const int32_t *cu_seqlens, int n_seq, gdr_dtype dtype, gdr_gate gate,
                           gdr_path path, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Gated DeltaNet-2 ("Gated DeltaNet-2, and the gate that was doing two jobs",
 * section "What decoupling actually means here"): the scalar step size splits
 * into an erase gate b_t (one value per key channel) and a write gate w_t (one
 * per value channel), e_t = b_t . k_t, z_t = w_t . v_t, and in the page's row
 * convention S_t = (I - k_t e_t^T) D_t S_{t-1} + k_t z_t^T.  In this library's
 * column convention (S is d_v x d_k):
 *     S' = S D_t;  u = z_t - S' e_t;  S <- S' + u k_t^T;  o_t = S q_t.
 * b = w = beta (broadcast) is gdr_fwd / gdr_decode_step.
 *
 * gdr_fwd_gdn2: the chunkwise prefill (that section's WY form: one triangular
 * solve serves both right-hand sides).
 *  q, k     [B, T, H, d_k]   dtype;  v, out [B, T, H, d_v] dtype
 *  g        [B, T, H] or [B, T, H, d_k]  fp32 log-decay
 *  b        [B, T, H, d_k]   fp32 erase gate;  w [B, T, H, d_v] fp32 write gate
 *  S0, S_final, cu_seqlens, n_seq, chunk, path, workspace: as for gdr_fwd.  The
 *  tensor-core path takes bf16 with d_k = d_v = 128 and chunk 64, with the
 *  per-channel decay (the page's setting) or a scalar one (broadcast over the
 *  key channels inside the kernel); everything else (chunk 16, 32, 64 or 128,
 *  d_k, d_v multiples of 16 up to 128) runs on the CUDA cores in fp32.
 *  gdr_fwd_gdn2_workspace_size gives the workspace (0 on the CUDA-core path).
 * gdr_decode_step_gdn2: one token per sequence in place on S_inout, with
 *  b [N, H, d_k] and w [N, H, d_v]; otherwise as gdr_decode_step.
 * Pointers are caller-owned device memory, 16-byte aligned; errors as gdr_fwd.
 */
size_t gdr_fwd_gdn2_workspace_size(int B, int T, int H, int d_k, int d_v, int chunk, int n_seq,
                                   int varlen, gdr_dtype dtype, gdr_gate gate, gdr_path path);
gdr_status gdr_fwd_gdn2(const void *q, const void *k, const void *v, const float *g,
                        const float *b, const float *w, const float *S0, void *out,
                        float *S_final, int B, int T, int H, int d_k, int d_v, int chunk,
                        const int32_t *cu_seqlens, int n_seq, gdr_dtype dtype, gdr_gate gate,
                        gdr_path path, void *workspace, size_t workspace_bytes, void *stream);
gdr_status gdr_decode_step_gdn2(const void *q, const void *k, const void *v, const float *g,
                                const float *b, const float *w, float *S_inout, void *out, int N,
                                int H, int d_k, int d_v, gdr_dtype dtype, gdr_gate gate,
                                void *stream);

/*
 * Implicit frame-level update ("video-delta-rule", sections "A First Attempt
 * at Frame-Level Updates" and "A Different Route").  The tokens of each
 * sequence form frames of n consecutive tokens (the last may be shorter).
 * Frame t has the erasure G_t = sum_i gamma_i k_i k_i^T and the write
 * C_t = sum_i gamma_i v_i k_i^T over its tokens, and the state takes the
 * backward-Euler step
 *     S_t (I + G_t) = S_{t-1} D_t + C_t
 * (D_t = the frame's decay, applied first); every query of frame t reads S_t:
 * o_i = S_t q_i.  The kernels form W_t = (I + G_t)^-1 (symmetric sweep, no
 * pivoting: every pivot of I + G_t is >= 1) and S_t = (S_{t-1} D_t + C_t) W_t;
 * n = 1 is the gated delta rule with step size gamma / (1 + gamma).
 *  q, k     [B, T, H, d_k]  dtype;  v, out [B, T, H, d_v]  dtype
 *  gamma    [B, T, H]       fp32 writing strength, >= 0 (a negative value can
 *                           make I + G_t indefinite: gdr_device_status then
 *                           reports GDR_ERR_INVALID)
 *  g        [B, F, H] or [B, F, H, d_k] fp32 log-decay per frame, F = ceil(T / n)
 *  S0       [B, H, d_v, d_k] fp32 or NULL (zero);  S_final likewise or NULL
 *  d_k a multiple of 16 in [16, 128]; d_v a multiple of 8 in [8, 128]
 *  workspace: gdr_fwd_frame_workspace_size(B, T, H, d_k, d_v, n) bytes,
 *           caller-owned device memory (per frame: G_t then W_t, C_t and S_t).
 * For bf16 with d_k = d_v = 128 the Gram and output passes run on the tensor
 * cores (bf16 operands, fp32 accumulation), and so does the chain, with each
 * product split into three bf16 products (x = x_hi + x_lo, A W ~ A_hi W_hi +
 * A_hi W_lo + A_lo W_hi) so that it keeps fp32 accuracy; the inverse is fp32
 * on the CUDA cores.  Otherwise every pass is fp32 on the CUDA cores.  Errors
 * as gdr_fwd.
 */
size_t gdr_fwd_frame_workspace_size(int B, int T, int H, int d_k, int d_v, int n);
gdr_status gdr_fwd_frame(const void *q, const void *k, const void *v, const float *g,
                         const float *gamma, const float *S0, void *out, float *S_final, int B,
                         int T, int H, int d_k, int d_v, int n, gdr_dtype dtype, gdr_gate gate,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdr_fwd_noalloc -- the prefill for callers that cannot allocate device
 * memory at call time (their memory manager owns the whole device heap and
 * forbids further cudaMalloc, or an allocation's device synchronisation is not
 * acceptable) and cannot pass a workspace of their own either.  The pages
 * have no counterpart of this entry point; it exists only for such callers.
 *
 * Same arguments and results as gdr_fwd with path GDR_PATH_TENSORCORE, minus
 * the workspace: the scratch comes from one fixed device array inside the
 * library, gdr_fwd_noalloc_scratch_bytes() bytes (32 MiB) large, which every
 * device that loads the library keeps until the process exits.  Calls whose
 * scratch need (gdr_fwd_workspace_size with GDR_PATH_TENSORCORE) exceeds it,
 * or whose shapes the tensor-core path does not take, return
 * GDR_ERR_UNSUPPORTED; nothing is allocated, ever.
 *
 * The first call on a device looks up the array's device address (a CUDA
 * runtime query, no allocation); make that first call outside any stream
 * capture.  All calls on a device share the one array and nothing in it needs
 * to start at zero, but two calls whose work overlaps on the GPU (different
 * streams, no ordering between them) race on it: order them.
 */
gdr_status gdr_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const float *S0, void *out, float *S_final, int B,
                           int T, int H, int d_k, int d_v, int chunk, const int32_t *cu_seqlens,
                           int n_seq, gdr_dtype dtype, gdr_gate gate, void *stream);
/* Size in bytes of the fixed scratch array used by gdr_fwd_noalloc. */
size_t gdr_fwd_noalloc_scratch_bytes(void);

/*
 * Range control of the tensor-core prefill's Gram weights.  Inside a chunk the
 * weights e^(G_l - G_m) of L and A (G = cumulative log-decay from the chunk
 * start; "Linear Attention, Visualized", sections "Gated DeltaNet (GDN) /
 * Complete per-chunk algorithm" and "Kimi Delta Attention (KDA) / Complete
 * per-chunk algorithm") are taken as e^(G_l - G_r) e^(G_r - G_m) around the
 * chunk's row r = 31, which keeps the Gram on the tensor cores.  A chunk in
 * which max_l |G_l - G_r| (any channel) reaches `limit` exponentiates every
 * difference instead (scalar gate: in the Gram epilogue; per-channel gate: L
 * and A summed on the CUDA cores); both give the same result up to rounding.
 * The default is 60; `limit` is clamped into [0, 80] (beyond 80 the factors
 * leave the normal fp32 / bf16 range) and 0 sends every chunk the exact way.
 * NaN leaves the setting unchanged.  Returns the previous limit.  Process-wide;
 * applies to calls made after it returns.
 */
float gdr_set_gram_spread_limit(float limit);

/*
 * Per-kernel launch accounting and timing (a small built-in profiler).
 * Kernel ids: GDR_K_DECODE, GDR_K_FWD_SIMT, GDR_K_TC_PLAN, GDR_K_TC_WY,
 * GDR_K_TC_STATE, GDR_K_GDP_REMAP (the Gated DeltaProduct expand/gather),
 * GDR_K_GDN2_SIMT and GDR_K_GDN2_DECODE (Gated DeltaNet-2), GDR_K_FRAME_GRAM,
 * GDR_K_FRAME_SOLVE, GDR_K_FRAME_CHAIN and GDR_K_FRAME_OUT (the implicit frame
 * update's passes).  Launches are always counted.  While timing is enabled,
 * every launch is bracketed by two CUDA events recorded on the launch's own
 * stream.  gdr_profile_read waits for the recorded events, returns the
 * launches and the summed device time (ms) of kernel `id` since the last read
 * of that id, and resets both.  Not thread-safe against concurrent gdr_* calls
 * from other host threads.
 */
enum { GDR_K_DECODE = 0, GDR_K_FWD_SIMT = 1, GDR_K_TC_PLAN = 2, GDR_K_TC_WY = 3,
       GDR_K_TC_STATE = 4, GDR_K_GDP_REMAP = 5, GDR_K_GDN2_SIMT = 6, GDR_K_GDN2_DECODE = 7,
       GDR_K_FRAME_GRAM = 8, GDR_K_FRAME_SOLVE = 9, GDR_K_FRAME_CHAIN = 10, GDR_K_FRAME_OUT = 11,
       GDR_K_COUNT = 12 };
void gdr_profile_enable(int on);
gdr_status gdr_profile_read(int id, long long *launches, double *total_ms);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H */
