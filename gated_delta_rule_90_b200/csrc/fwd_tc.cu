// Tensor-core chunkwise prefill of the gated delta rule (sm_100a: tcgen05 MMA
// with TMEM accumulators, operands staged in shared memory by TMA).
//
// Shapes: bf16 q, k, v, out; d_k = d_v = 128; chunk C = 64; fp32 g, beta, states.
// The chunkwise form is that of "Linear Attention, Visualized", sections
// "Gated DeltaNet (GDN) / Complete per-chunk algorithm" and "Kimi Delta
// Attention (KDA) / Complete per-chunk algorithm", in the column convention
// (S is d_v x d_k).  Two kernels:
//
//  wy_kernel     one CTA per (chunk, head), all chunks in parallel (the pages
//                note that the local quantities of every chunk are independent):
//                  G = cumsum(g);  [K;Q] K^T on the tensor cores (Gram, M = 128);
//                  L = tril_-1(K K^T . Gamma), A = tril_0(Q K^T . Gamma);
//                  (I + diag(beta) L) T = diag(beta) by column forward
//                  substitution in fp32 (shared memory);
//                  U^T = V^T T^T and W<-^T = K<-^T T^T on the tensor cores;
//                  (W<- is stored back in token-major order)
//                writes W<-, U, A, Q<- = e^G . q, K-> = e^(G_C - G) . k and the
//                chunk decay e^(G_C) to the workspace (bf16 tiles, fp32 decay).
//  state_kernel  one CTA per (sequence, head), chunks in order (the boundary
//                pass).  S (d_v x d_k fp32) lives in TMEM for the whole
//                sequence; per chunk:
//                  Z^T = U^T - S W<-^T,      O^T = S Q<-^T + Z^T A^T,
//                  S <- S Diag(e^(G_C)) + Z^T K->,
//                four GEMMs with M = d_v = 128 on the tensor cores; the next
//                chunk's tiles are prefetched by TMA into a second stage.
//
// Per-channel gates (KDA) enter the Gram GEMM factorised around the middle
// row r = 31 of the chunk: (k_l . e^(G_l - G_r)) . (k_m . e^(G_r - G_m)), so
// every factor stays within e^(|G_l - G_r|) of 1 -- never a ratio of products.
// That needs |G_l - G_r| well inside the fp32/bf16 exponent range.  A chunk in
// which some channel's spread max_l |G_l - G_r| reaches the limit (60 by
// default) takes the exact route instead: L and A are summed on the CUDA cores
// with e^(G_lc - G_mc) exponentiated per element (never above 1 for a decay),
// and Q<-, K->, K<- use e^(G), e^(G_C - G) directly.
//
// Tokens of a chunk that runs past the end of its sequence are zeroed in
// shared memory (k = q = v = 0, beta = 0, g = 0), which leaves every valid row
// unchanged.  Every wait on an mbarrier is bounded: on expiry the kernel
// records a timeout in the device error word, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace gdr {
namespace tc {

using namespace sm100;

constexpr int C = 64;
constexpr int D = 128;
constexpr uint32_t kSpin = 1u << 24;  // poll limit of every mbarrier wait

constexpr uint32_t kTileBytes = C * D * 2;   // 16 KB: one [64][128] bf16 tile
constexpr uint32_t kHalfBytes = C * 64 * 2;  // 8 KB: one [64][64] bf16 atom column
constexpr uint32_t kDecBytes = D * 4;

struct Geo {
    int B, T, H, n_seq, nc;  // nc: chunks per sequence (regular batches)
    int varlen, T_total, n_slots;
    // > 1: the rows are a Gated DeltaProduct virtual sequence with keep
    // substeps per token; out has one row per token and receives the last
    // substep's output only
    int keep;
    // largest within-chunk |G_l - G_31| (cumulative log-decay, any channel)
    // for which the Gram weights e^(G_l - G_m) are taken as the product of two
    // per-row factors; a chunk beyond it exponentiates every difference
    float spread_limit;
};

struct Ws {
    int *chunk_start;  // [n_seq + 1] (varlen)
    int *order;        // [n_seq] longest first (varlen)
    float *dec;        // [slots*H][128]
    __nv_bfloat16 *W;              // [slots*H][64 (token)][128 (d)]
    __nv_bfloat16 *U;              // transposed: [slots*H][128 (d)][64 (token)]
    __nv_bfloat16 *Q, *K;          // [slots*H][64 (token)][128 (d)]
    __nv_bfloat16 *A;              // [slots*H][64][64]
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return (uint8_t *)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

// bf16x8 <-> float8 helpers (16-byte chunks of a tile)
__device__ __forceinline__ bool locate_chunk(const Geo &geo, const int32_t *cu, const Ws &ws,
                                             int gcid, long &tstart, int &len) {
    long t0, t1;
    int s, cidx;
    if (geo.varlen) {
        const int total = ws.chunk_start[geo.n_seq];
        if (gcid >= total) return false;
        int lo = 0, hi = geo.n_seq - 1;  // last s with chunk_start[s] <= gcid
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (ws.chunk_start[mid] <= gcid) lo = mid; else hi = mid - 1;
        }
        s = lo;
        cidx = gcid - ws.chunk_start[s];
    } else {
        s = gcid / geo.nc;
        cidx = gcid % geo.nc;
    }
    seq_bounds(cu, s, geo.T, geo.T_total, t0, t1);
    tstart = t0 + (long)cidx * C;
    len = (int)min((long)C, t1 - tstart);
    return len > 0;
}

// ------------------------------------------------------------------ plan (varlen)
// One CTA: per-sequence chunk counts, their prefix sum and a longest-first order.
__global__ void plan_kernel(const int32_t *cu, int n_seq, int T_total, int *chunk_start,
                            int *order) {
    for (int s = threadIdx.x; s < n_seq; s += blockDim.x) {
        long t0, t1;
        seq_bounds(cu, s, 0, T_total, t0, t1);
        chunk_start[s + 1] = (int)((t1 - t0 + C - 1) / C);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        chunk_start[0] = 0;
        for (int s = 0; s < n_seq; ++s) chunk_start[s + 1] += chunk_start[s];
    }
    __syncthreads();
    // rank sort by length (descending, ties by index); identity beyond 4096 sequences
    for (int s = threadIdx.x; s < n_seq; s += blockDim.x) {
        if (n_seq > 4096) {
            order[s] = s;
            continue;
        }
        long a0, a1;
        seq_bounds(cu, s, 0, T_total, a0, a1);
        const long ls = a1 - a0;
        int rank = 0;
        for (int o = 0; o < n_seq; ++o) {
            long b0, b1;
            seq_bounds(cu, o, 0, T_total, b0, b1);
            const long lo = b1 - b0;
            rank += (lo > ls) || (lo == ls && o < s);
        }
        order[rank] = s;
    }
}

// Sums each of v[0..7] over the 32 lanes of a warp in 9 shuffles (each step
// halves the values a lane keeps); lane L returns the total of v[(L >> 2) & 7].
__device__ __forceinline__ float warp_sum8(const float (&v)[8], int lane) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    float w[4], x[2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = (b4 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, b4 ? v[i] : v[i + 4], 16);
#pragma unroll
    for (int i = 0; i < 2; ++i)
        x[i] = (b3 ? w[i + 2] : w[i]) + __shfl_xor_sync(0xffffffffu, b3 ? w[i] : w[i + 2], 8);
    float y = (b2 ? x[1] : x[0]) + __shfl_xor_sync(0xffffffffu, b2 ? x[0] : x[1], 4);
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 2);
    return y;
}
// Four consecutive bf16 of a 128-byte-swizzled [rows][64] atom: row r,
// columns 4 q .. 4 q + 3 (q = 0..15).
__device__ __forceinline__ void ld4_sw128(const uint8_t *atom, int r, int q, float *f) {
    const uint2 u = *reinterpret_cast<const uint2 *>(atom + r * 128 + (((q >> 1) ^ (r & 7)) << 4) +
                                                     (q & 1) * 8);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}

// ------------------------------------------------------------------ WY kernel
// 256 threads, 128 TMEM columns.  For accumulator epilogues, warp w serves TMEM
// lane quadrant (w & 3) and column half (w >> 2).
constexpr int kWyThreads = 256;
constexpr uint32_t kWyTmemCols = 128;
// Issues every TMA load and the A store: a thread outside warps 0-1, which
// load the gates and run the diagonal-block solve, so that a slow TMA issue
// never holds up that work.
constexpr int kWyTmaThread = 128;

// Shared-memory plan (byte offsets from a 1024-aligned base).  Regions are
// reused once their first contents are dead, so a CTA needs 74 KB and three
// fit on an SM, for either gate:
//   KQ  [0, 32K)     raw K (rows 0-63) and Q (rows 64-127) in two 128-byte atom
//                    columns (per-channel gate: K^ and Q^ in place); V replaces Q
//                    once the Gram has read it.  At the end: U^T staging.
//   TT  [32K, 40K)   per-channel gate: the rows R, G_C and e^(G_C - R) until the
//                    Gram; then A staging for its TMA store, then T.
//   NT  [40K, 56K)   N^T fp32 [64][64]; after the solve, K<- (bf16, 2 atoms).
//                    Per-channel gate: NT and XR first hold the gate tile G, then
//                    NT holds K-check (the Gram's B operand).
//   XR  [56K, 72.3K) X fp32 [64][65].
//   then the small region: scalar gate G and beta per row; per-channel gate beta
//   and e^R per channel; two mbarriers and the TMEM slot.  The scalar gate's Gram
//   factors e^(G - R), e^(R - G) and their flag live in XR, dead until the solve.
struct WySmem {
    static constexpr uint32_t KQ = 0, TT = 32768, NT = 40960, XR = 57344;
    static constexpr int NTS = 64;                                   // N^T row stride (floats)
    static constexpr int XST = 65;                                   // X row stride (floats)
    static constexpr uint32_t XEND = XR + 64 * XST * 4;
    static constexpr uint32_t small(bool) { return XEND; }
    static constexpr int small_floats(bool ch) { return ch ? 64 + D : 128; }
    static constexpr uint32_t small_bytes(bool ch) { return small_floats(ch) * 4 + 64; }
};

// SUB: the chunk size of the method, 64 or 16.  With 16 a
// 64-token tile holds four chunks: G restarts every 16 rows, L, A and T are
// block diagonal (the 16 x 16 diagonal blocks of the 64 x 64 solve), K->
// decays to each chunk's own end, and four decay rows are written.  The
// per-channel Gram then factorises around each chunk's start (G = 0), so the
// reading factor e^G is K<-'s own and only the chunk ends G_C are tabulated.
// DEC (per-channel decay only): Gated DeltaNet-2's erase gate b and write gate
// w replace beta ("Gated DeltaNet-2, and the gate that was doing two jobs",
// section "What decoupling actually means here"): the Gram's reading rows are
// e = b . k (so L = tril_-1(E K^T . Gamma) and W<- = T E<-), T solves
// (I + L) T = I, and U = T (w . V).  The writing direction stays k (K->, A).
// BC (with CH): the decay is one scalar per token, broadcast over the key
// channels of the gate tile in shared memory instead of loaded per channel.
template <bool CH, bool DEC = false, bool BC = false, int SUB = C>
__global__ void __launch_bounds__(kWyThreads, CH ? 3 : 0)
wy_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
          const __grid_constant__ CUtensorMap tm_Ust,
          const __grid_constant__ CUtensorMap tm_Ast, const float *__restrict__ g,
          const float *__restrict__ beta, const float *__restrict__ eg,
          const float *__restrict__ wg, const int32_t *__restrict__ cu, Geo geo, Ws ws,
          unsigned int *err) {
    constexpr int NTS = WySmem::NTS, XST = WySmem::XST;
    constexpr bool SUB16 = SUB == 16;
    static_assert(SUB == C || SUB == 16, "method chunk of 64 or 16 tokens");
    // same method chunk: m and l in one SUB-row block
    auto same = [](int m, int l) { return !SUB16 || (m >> 4) == (l >> 4); };
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint8_t *sKQ = sm + WySmem::KQ, *sT = sm + WySmem::TT;
    uint8_t *sKL = sm + WySmem::NT;                                    // after the solve
    uint8_t *sV = sKQ + 8192;                                          // Q's place, after the Gram
    uint8_t *sKC = sm + WySmem::NT;                                    // per-channel gate only
    float *sN = reinterpret_cast<float *>(sm + WySmem::NT);            // N^T [m][l]
    float *sX = reinterpret_cast<float *>(sm + WySmem::XR);            // X [row][col]
    float *sGt = reinterpret_cast<float *>(sm + WySmem::NT);           // per-channel G [64][128]
    float *sSm = reinterpret_cast<float *>(sm + WySmem::small(CH));
    float *sTf = reinterpret_cast<float *>(sm + WySmem::TT);
    float *sG = CH ? sTf : sSm;                                        // scalar: G [64]; channel: R row [128]
    float *sGC = sTf + D;                                              // channel: G_C row [128]
    float *sB = CH ? sSm : sSm + 64;                                   // beta [64]
    // exponential tables, so that no element-wise exp is needed below
    float *eR = sSm + 64, *eCR = sTf + 2 * D;                          // channel: per channel
    float *sGC4 = sTf, *eCR4 = sTf + 4 * D;  // channel, 16-token chunks: G_C, e^(G_C) [4][128]
    float *eA = sX, *eB = sX + 64;                                     // scalar: per row (XR)
    int *sFact = reinterpret_cast<int *>(sX + 128);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sSm + WySmem::small_floats(CH));  // [2]
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, hf = warp >> 2;
    const uint32_t lb = (uint32_t)(qd * 32) << 16;
    const int gcid = blockIdx.x, h = blockIdx.y;
    long tstart;
    int len;
    if (!locate_chunk(geo, cu, ws, gcid, tstart, len)) return;  // whole CTA, before any sync
    const size_t slot = (size_t)gcid * geo.H + h;
    const int x0 = h * D, ytok = (int)tstart;
    if (kChecked) {  // checked build: the chunk's tokens, its workspace slot, the TMA boxes
        const long long rows = geo.varlen ? (long long)geo.T_total : (long long)geo.B * geo.T;
        const long long xe = (long long)geo.H * D;
        if (!(chk_span(tstart, len, rows, err) &&
              chk_span((long long)slot, 1, (long long)geo.n_slots * geo.H, err) &&
              chk_tma(x0, ytok, 2, xe, rows, err) && chk_tma(x0 + 64, ytok, 2, xe, rows, err)))
            return;  // whole CTA, before any sync
    }

    // The TMA thread initialises the barriers and issues the loads first, so
    // that their latency overlaps the TMEM allocation and the gate loads.
    if (tid == kWyTmaThread) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        mbar_arrive_expect_tx(&bars[0], 4 * kHalfBytes + (CH && !BC ? C * D * 4 : 0));
        tma_load_2d(sKQ, &tm_k, &bars[0], x0, ytok);
        tma_load_2d(sKQ + 16384, &tm_k, &bars[0], x0 + 64, ytok);
        tma_load_2d(sKQ + 8192, &tm_q, &bars[0], x0, ytok);
        tma_load_2d(sKQ + 16384 + 8192, &tm_q, &bars[0], x0 + 64, ytok);
        if (CH && !BC) tma_load_2d(sGt, &tm_g, &bars[0], x0, ytok);  // [64][128] fp32 per-channel gates
    }
    if (warp == 0) {
        tmem_alloc(tslot, kWyTmemCols);
        tmem_relinquish();
    }
    // gates and beta (zero beyond the sequence end), cumulative log-decay G
    if (!CH && tid < C) sG[tid] = (tid < len) ? g[(size_t)(tstart + tid) * geo.H + h] : 0.f;
    if (tid < C) sB[tid] = (tid < len) ? (DEC ? 1.f : beta[(size_t)(tstart + tid) * geo.H + h]) : 0.f;
    if (BC) {  // the gate tile from one log-decay per token
        for (int e = tid; e < C * D / 4; e += kWyThreads) {
            const int l = e / (D / 4);
            const float gl = (l < len) ? g[(size_t)(tstart + l) * geo.H + h] : 0.f;
            reinterpret_cast<float4 *>(sGt)[e] = make_float4(gl, gl, gl, gl);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    // per-channel gate: this chunk takes the exact route (see the file header)
    int fb = 0;
    if (!CH && warp == 0) {
        // rows 0-31 in a, 32-63 in b; 16-token chunks scan each 16-row block
        float a = sG[lane], b = sG[lane + 32];
#pragma unroll
        for (int off = 1; off < (SUB16 ? 16 : 32); off <<= 1) {
            const float ya = __shfl_up_sync(0xffffffffu, a, off);
            const float yb = __shfl_up_sync(0xffffffffu, b, off);
            if ((SUB16 ? (lane & 15) : lane) >= off) {
                a += ya;
                b += yb;
            }
        }
        if (!SUB16) b += __shfl_sync(0xffffffffu, a, 31);
        sG[lane] = a;
        sG[lane + 32] = b;
        // Gamma[l][m] = e^(G_l - G_m) factorised around a middle row R (row 31,
        // or row 7 of each 16-row chunk) as e^(G_l - R) e^(R - G_m) -- exact up
        // to rounding while every |G_l - R| stays far from the fp32 exp range;
        // otherwise the Gram epilogue takes the exp of each difference (flag 0)
        const float Ra = __shfl_sync(0xffffffffu, a, SUB16 ? ((lane & 16) | 7) : 31);
        const float Rb = SUB16 ? __shfl_sync(0xffffffffu, b, (lane & 16) | 7) : Ra;
        float spread = fmaxf(fabsf(a - Ra), fabsf(b - Rb));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            spread = fmaxf(spread, __shfl_xor_sync(0xffffffffu, spread, off));
        eA[lane] = __expf(a - Ra);
        eA[lane + 32] = __expf(b - Rb);
        eB[lane] = __expf(Ra - a);
        eB[lane + 32] = __expf(Rb - b);
        if (lane == 0) *sFact = spread < geo.spread_limit;
    }
    {
        const bool ok_ld = mbar_wait_bounded(&bars[0], 0, kSpin, err);
        if (!__syncthreads_and(ok_ld)) goto cleanup;
    }
    if (CH) {
        // per-channel scan, rows past the sequence end count as g = 0: thread
        // (c, half) scans 32 rows, the upper half then adds the lower half's total
        const int c = tid & 127, r0 = (tid >> 7) * 32;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = (r0 + i < len) ? sGt[(r0 + i) * D + c] : 0.f;
#pragma unroll
        for (int i = 1; i < 32; ++i)
            if (!SUB16 || i != 16) v[i] += v[i - 1];  // 16-token chunks restart at row 16
        // spread = max_l |G_l - R| of this channel (R = G_31; for 16-token
        // chunks R = 0, the chunk's start)
        float spread = 0.f;
        if (!r0) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                sGt[i * D + c] = v[i];
                spread = fmaxf(spread, fabsf(v[i] - (SUB16 ? 0.f : v[31])));
            }
        }
        __syncthreads();
        if (r0) {
            const float base = SUB16 ? 0.f : sGt[31 * D + c];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                sGt[(32 + i) * D + c] = v[i] + base;
                spread = fmaxf(spread, fabsf(v[i]));
            }
        }
        fb = __syncthreads_or(!(spread < geo.spread_limit));
        if (SUB16) {  // each chunk's G_C and decay e^(G_C)
            for (int e = tid; e < (C / 16) * D; e += kWyThreads) {
                const float GC = sGt[((e / D) * 16 + 15) * D + (e % D)];
                sGC4[e] = GC;
                eCR4[e] = __expf(GC);
            }
        } else if (tid < D) {
            const float R = sGt[31 * D + tid], GC = sGt[(C - 1) * D + tid];
            sG[tid] = R;    // reference row R of the Gram factorisation
            sGC[tid] = GC;  // G_C
            eR[tid] = __expf(R);
            eCR[tid] = __expf(GC - R);
        }
    }
    // zero K and Q rows beyond the sequence end (whole 128-byte rows)
    if (len < C) {
        for (int e = tid; e < (C - len) * 8 * 4; e += kWyThreads) {
            const int r = len + e / 32, part = e % 32, tile = part >> 3, ch16 = part & 7;
            uint8_t *base = sKQ + (tile & 1) * 16384 + (tile >> 1) * 8192;
            *reinterpret_cast<uint4 *>(base + r * 128 + ch16 * 16) = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    // From the raw K and Q: Q<- = e^G . q and K-> = e^(G_C - G) . k to the
    // workspace; per-channel gate also K-check = k e^(R - G) and, in place,
    // K^ = k e^(G - R), Q^ = q e^(G - R) (R = row 31 of G).
    {
        // thread: channels c0..c0+7 (8-channel group cg) of rows l0, l0+16, ...;
        // the group's per-channel factors stay in registers
        __nv_bfloat16 *Qg = ws.Q + slot * (C * D), *Kg = ws.K + slot * (C * D);
        const int cg = tid & 15, c0 = cg * 8, a = cg >> 3, l0 = tid >> 4;
        float R8[8], eR8[8], eCR8[8];
        uint4 kcv[C / 16];  // per-channel gate: K-check, stored once G is read
        if (CH && SUB16) {  // R = 0: e^R = 1; e^(G_C - R) per chunk, below
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                R8[i] = 0.f;
                eR8[i] = 1.f;
            }
        } else if (CH) {
            ld8(sG + c0, R8);
            ld8(eR + c0, eR8);
            ld8(eCR + c0, eCR8);
        }
#pragma unroll
        for (int k = 0; k < C / 16; ++k) {
            if (CH && SUB16) ld8(eCR4 + k * D + c0, eCR8);  // row l is in chunk k
            const int l = l0 + 16 * k, j = (cg & 7) ^ (l & 7);  // physical 16-byte chunk
            const uint32_t off = a * 16384 + l * 128 + j * 16;
            float kv[8], qv[8], wq[8], wk[8];
            unpack8(*reinterpret_cast<const uint4 *>(sKQ + off), kv);
            unpack8(*reinterpret_cast<const uint4 *>(sKQ + off + 8192), qv);
            if (CH) {
                float kh[8], qh[8], kc[8], G8[8], b8[8];
                ld8(sGt + l * D + c0, G8);
                if (DEC) {  // erase gate of this row (reading side)
                    const size_t gro = ((size_t)(tstart + l) * geo.H + h) * D + c0;
                    if (l < len) {
                        ld8(eg + gro, b8);
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) b8[i] = 0.f;
                    }
                }
                if (fb) {  // exact route: e^G and e^(G_C - G) themselves (at most 1)
                    float GC8[8];
                    ld8(SUB16 ? sGC4 + k * D + c0 : sGC + c0, GC8);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        wq[i] = qv[i] * __expf(G8[i]);
                        wk[i] = kv[i] * __expf(GC8[i] - G8[i]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        // e^G = e^(G - R) e^R and e^(G_C - G) = e^(R - G) e^(G_C - R)
                        const float e1 = __expf(G8[i] - R8[i]), e2 = __expf(R8[i] - G8[i]);
                        wq[i] = qv[i] * (e1 * eR8[i]);
                        wk[i] = kv[i] * (e2 * eCR8[i]);
                        kh[i] = (DEC ? kv[i] * b8[i] : kv[i]) * e1;
                        qh[i] = qv[i] * e1;
                        kc[i] = kv[i] * e2;
                    }
                    *reinterpret_cast<uint4 *>(sKQ + off) = pack8(kh);
                    *reinterpret_cast<uint4 *>(sKQ + off + 8192) = pack8(qh);
                    kcv[k] = pack8(kc);
                }
            } else {
                const float eq = __expf(sG[l]), ek = __expf(sG[SUB16 ? (l | 15) : C - 1] - sG[l]);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    wq[i] = qv[i] * eq;
                    wk[i] = kv[i] * ek;
                }
            }
            *reinterpret_cast<uint4 *>(Qg + l * D + c0) = pack8(wq);
            *reinterpret_cast<uint4 *>(Kg + l * D + c0) = pack8(wk);
        }
        if (SUB16) {  // one decay row per 16-token chunk
            for (int e = tid; e < (C / 16) * D; e += kWyThreads)
                ws.dec[slot * (C / 16) * D + e] = CH ? eCR4[e] : __expf(sG[(e / D) * 16 + 15]);
        } else if (tid < D) {
            ws.dec[slot * D + tid] = CH ? (fb ? __expf(sGC[tid]) : eCR[tid] * eR[tid])
                                        : __expf(sG[C - 1]);
        }
        if (CH && !fb) {  // the gate tile is read: K-check takes its first half
            __syncthreads();
#pragma unroll
            for (int k = 0; k < C / 16; ++k) {
                const int l = l0 + 16 * k, j = (cg & 7) ^ (l & 7);
                *reinterpret_cast<uint4 *>(sKC + a * 8192 + l * 128 + j * 16) = kcv[k];
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    if (!fb) {
        // Gram: TMEM[0:64) = [K;Q] (128 x 128) * Kc^T (64 x 128)^T
        if (tid == 0) {
            tc_fence_after();
            const uint8_t *Bb = CH ? sKC : sKQ;
            const uint32_t bstride = CH ? 8192 : 16384;
            const uint32_t id = idesc_bf16(128, 64, 0, 0);
            const uint64_t ad = sdesc_sw128(smem_u32(sKQ), 16, 1024);
            const uint64_t bd = sdesc_sw128(smem_u32(Bb), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk & 3) * 32;
                mma_bf16_ss(tmem, sdesc_add(ad, (kk >> 2) * 16384 + koff),
                            sdesc_add(bd, (kk >> 2) * bstride + koff), id, kk > 0);
            }
            mma_commit(&bars[1]);
        }
        {
            const bool ok = mbar_wait_bounded(&bars[1], 0, kSpin, err);
            if (!__syncthreads_and(ok)) goto cleanup;
        }
        tc_fence_after();
        {
            // accumulator rows 0..63: K K^T -> N = diag(beta) tril_-1(. Gamma), stored
            // transposed; rows 64..127: Q K^T -> A = tril_0(. Gamma), bf16, staged in TT
            const int l = (qd & 1) * 32 + lane, m0 = hf * 32;
            float gr[32];
            tmem_ld16(tmem + lb + m0, gr);
            tmem_ld16(tmem + lb + m0 + 16, gr + 16);
            tmem_wait_ld();
            // gam(m) = Gamma[l][m] (scalar gate; the per-channel gate is inside the operands)
            auto epilogue = [&](auto gam) {
                if (qd < 2) {
                    const float bl = sB[l];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int m = m0 + i;
                        sN[m * NTS + l] = (m < l && same(m, l)) ? bl * gr[i] * gam(m) : 0.f;
                    }
                } else {
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        float o[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int m = m0 + jj * 8 + i;
                            o[i] = (m <= l && same(m, l)) ? gr[jj * 8 + i] * gam(m) : 0.f;
                        }
                        const int j = hf * 4 + jj;
                        *reinterpret_cast<uint4 *>(sT + l * 128 + ((j ^ (l & 7)) << 4)) = pack8(o);
                    }
                }
            };
            if (CH) {
                epilogue([](int) { return 1.f; });
            } else if (*sFact) {
                const float eAl = eA[l];
                epilogue([&](int m) { return eAl * eB[m]; });
            } else {
                const float Gl = sG[l];
                epilogue([&](int m) { return __expf(Gl - sG[m]); });
            }
        }
    } else {
        // Exact route (per-channel gate, a chunk beyond the spread limit): L and
        // A on the CUDA cores with every weight e^(G_lc - G_mc) exponentiated.
        // A warp takes (row l, columns m0..m0+3) at a time, its lanes four
        // channels each; beta L goes to the W tile of the workspace (fp32,
        // N^T order) until the gate tile is dead, A straight to its workspace
        // tile.
        float *Nsc = reinterpret_cast<float *>(ws.W + slot * (C * D));
        __nv_bfloat16 *Ag = ws.A + slot * (C * C);
        for (int e = tid; e < C * C; e += kWyThreads)
            if (e % C > e / C || !same(e % C, e / C)) Ag[e] = __float2bfloat16_rn(0.f);
        const int qa = lane >> 4, qc = lane & 15;  // atom, 4-channel group
        int gi = 0;
        for (int l = 0; l < C; ++l) {
            for (int m0 = SUB16 ? (l & ~15) : 0; m0 <= l; m0 += 4, ++gi) {
                if ((gi & 7) != warp) continue;
                const float4 gl = *reinterpret_cast<const float4 *>(sGt + l * D + 4 * lane);
                float el[4], ql[4], acc[8];
                ld4_sw128(sKQ + qa * 16384, l, qc, el);
                ld4_sw128(sKQ + qa * 16384 + 8192, l, qc, ql);
                if (DEC) {  // reading row e = b . k (zero beyond the sequence end)
                    const float4 bb = (l < len)
                        ? *reinterpret_cast<const float4 *>(
                              eg + ((size_t)(tstart + l) * geo.H + h) * D + 4 * lane)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    el[0] *= bb.x; el[1] *= bb.y; el[2] *= bb.z; el[3] *= bb.w;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int m = min(m0 + u, C - 1);  // m > l: computed, never stored
                    const float4 gm = *reinterpret_cast<const float4 *>(sGt + m * D + 4 * lane);
                    float km[4];
                    ld4_sw128(sKQ + qa * 16384, m, qc, km);
                    const float w0 = __expf(gl.x - gm.x) * km[0], w1 = __expf(gl.y - gm.y) * km[1];
                    const float w2 = __expf(gl.z - gm.z) * km[2], w3 = __expf(gl.w - gm.w) * km[3];
                    acc[u] = el[0] * w0 + el[1] * w1 + el[2] * w2 + el[3] * w3;
                    acc[4 + u] = ql[0] * w0 + ql[1] * w1 + ql[2] * w2 + ql[3] * w3;
                }
                const float tot = warp_sum8(acc, lane);
                if ((lane & 3) == 0) {
                    const int vi = lane >> 2;
                    if (vi < 4) {
                        const int m = m0 + vi;
                        if (m < l) Nsc[m * C + l] = sB[l] * tot;
                    } else {
                        const int m = m0 + vi - 4;
                        if (m <= l) Ag[l * C + m] = __float2bfloat16_rn(tot);
                    }
                }
            }
        }
        __syncthreads();
        // K<- = e^G . k (. b) over the raw K rows, while the gate tile lives
        {
            const int cg = tid & 15, c0 = cg * 8, a = cg >> 3, l0 = tid >> 4;
#pragma unroll
            for (int k = 0; k < C / 16; ++k) {
                const int l = l0 + 16 * k, j = (cg & 7) ^ (l & 7);
                const uint32_t off = a * 16384 + l * 128 + j * 16;
                float kv[8], G8[8], o[8];
                unpack8(*reinterpret_cast<const uint4 *>(sKQ + off), kv);
                ld8(sGt + l * D + c0, G8);
                if (DEC) {
                    float b8[8];
                    if (l < len) {
                        ld8(eg + ((size_t)(tstart + l) * geo.H + h) * D + c0, b8);
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) b8[i] = 0.f;
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) kv[i] *= b8[i];
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) o[i] = kv[i] * __expf(G8[i]);
                *reinterpret_cast<uint4 *>(sKQ + off) = pack8(o);
            }
        }
        __syncthreads();  // the gate tile is dead: N^T into its place
        for (int e = tid; e < C * C; e += kWyThreads) {
            const int m = e / C, l = e % C;
            sN[m * NTS + l] = (m < l && same(m, l)) ? Nsc[e] : 0.f;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == kWyTmaThread) {  // A -> workspace (the exact route stored it already)
        if (!fb) {
            tma_store_2d(&tm_Ast, sT, 0, (int)(slot * C));
            bulk_commit_group();
        }
        // Q is read: V takes its place (lands during the solve)
        mbar_arrive_expect_tx(&bars[0], 2 * kHalfBytes);
        tma_load_2d(sV, &tm_v, &bars[0], x0, ytok);
        tma_load_2d(sV + 16384, &tm_v, &bars[0], x0 + 64, ytok);
    }
    // T = (I + N)^{-1} diag(beta), N = diag(beta) L strictly lower, by 16 x 16
    // blocks: X_ii = (I + N_ii)^{-1} by forward substitution (one column per
    // thread); then X_10, X_32 and finally the lower-left 32 x 32 quadrant.
    {
        if (tid < C) {
            const int b = tid >> 4, j = tid & 15;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float p0 = 0.f, p1 = 0.f;
#pragma unroll
                for (int m = 0; m < i; ++m) {  // N_bb[i][m] = N^T[16b+m][16b+i]
                    const float nv = sN[(16 * b + m) * NTS + 16 * b + i];
                    if (m & 1) p1 = fmaf(nv, x[m], p1);
                    else p0 = fmaf(nv, x[m], p0);
                }
                x[i] = ((i == j) ? 1.f : 0.f) - (p0 + p1);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) sX[(16 * b + i) * XST + 16 * b + j] = x[i];
        }
        __syncthreads();
        if (SUB16) {  // block diagonal: the diagonal blocks are the whole inverse
            if (tid == kWyTmaThread) bulk_wait_group_read<0>();  // the A staging is read
            __syncthreads();
        } else {
            // tasks: strips of 4 rows x 1 column of a 16 x 16 block (float4 over N^T rows)
            const int c = tid & 15, r0 = ((tid >> 4) & 3) * 4, blk = tid >> 6;
            {   // level A: X_10 = -X_11 (N_10 X_00), X_32 = -X_33 (N_32 X_22)
                const int j = blk * 2, i = j + 1;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                if (tid < 128) {
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float xv = sX[(16 * j + m) * XST + 16 * j + c];
                        const float4 nv = *reinterpret_cast<const float4 *>(sN + (16 * j + m) * NTS + 16 * i + r0);
                        acc[0] = fmaf(nv.x, xv, acc[0]);
                        acc[1] = fmaf(nv.y, xv, acc[1]);
                        acc[2] = fmaf(nv.z, xv, acc[2]);
                        acc[3] = fmaf(nv.w, xv, acc[3]);
                    }
#pragma unroll
                    for (int t = 0; t < 4; ++t) sX[(16 * i + r0 + t) * XST + 16 * j + c] = acc[t];
                }
                __syncthreads();
                float res[4] = {0.f, 0.f, 0.f, 0.f};
                if (tid < 128) {
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float pv = sX[(16 * i + m) * XST + 16 * j + c];
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            res[t] = fmaf(sX[(16 * i + r0 + t) * XST + 16 * i + m], pv, res[t]);
                    }
                }
                __syncthreads();
                if (tid < 128) {
#pragma unroll
                    for (int t = 0; t < 4; ++t) sX[(16 * i + r0 + t) * XST + 16 * j + c] = -res[t];
                }
                __syncthreads();
            }
            {   // level B: P_ij = N_i0 X_0j + N_i1 X_1j (i in {2,3}, j in {0,1});
                // X_2j = -X_22 P_2j,  X_3j = -(X_32 P_2j + X_33 P_3j)
                const int i = 2 + (blk >> 1), j = blk & 1;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                for (int kb = j; kb < 2; ++kb) {
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float xv = sX[(16 * kb + m) * XST + 16 * j + c];
                        const float4 nv = *reinterpret_cast<const float4 *>(sN + (16 * kb + m) * NTS + 16 * i + r0);
                        acc[0] = fmaf(nv.x, xv, acc[0]);
                        acc[1] = fmaf(nv.y, xv, acc[1]);
                        acc[2] = fmaf(nv.z, xv, acc[2]);
                        acc[3] = fmaf(nv.w, xv, acc[3]);
                    }
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) sX[(16 * i + r0 + t) * XST + 16 * j + c] = acc[t];
                __syncthreads();  // N^T is dead from here on
                float res[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < 16; ++m) {  // X_ii P_ij
                    const float pv = sX[(16 * i + m) * XST + 16 * j + c];
#pragma unroll
                    for (int t = 0; t < 4; ++t)
                        res[t] = fmaf(sX[(16 * i + r0 + t) * XST + 16 * i + m], pv, res[t]);
                }
                if (i == 3) {
#pragma unroll
                    for (int m = 0; m < 16; ++m) {  // + X_32 P_2j
                        const float pv = sX[(32 + m) * XST + 16 * j + c];
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            res[t] = fmaf(sX[(48 + r0 + t) * XST + 32 + m], pv, res[t]);
                    }
                }
                if (tid == kWyTmaThread) bulk_wait_group_read<0>();  // the A staging is read
                __syncthreads();
#pragma unroll
                for (int t = 0; t < 4; ++t) sX[(16 * i + r0 + t) * XST + 16 * j + c] = -res[t];
                __syncthreads();
            }
        }
        // T[i][j] = X[i][j] beta_j (lower triangle) -> bf16, K-major SW128 tile
        for (int e = tid; e < C * 8; e += kWyThreads) {
            const int i = e >> 3, j8 = e & 7;
            float o[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j8 * 8 + u;
                o[u] = (j <= i && same(j, i)) ? sX[i * XST + j] * sB[j] : 0.f;
            }
            *reinterpret_cast<uint4 *>(sT + i * 128 + ((j8 ^ (i & 7)) << 4)) = pack8(o);
        }
        // K<- into the dead N^T area: scalar gate e^G . k from raw K, per-channel
        // gate K^ . e^R (exact route: K<- is already in place)
        {
            const int cg = tid & 15, c0 = cg * 8, a = cg >> 3, l0 = tid >> 4;
            float eR8[8];
            if (CH && SUB16) {
#pragma unroll
                for (int i = 0; i < 8; ++i) eR8[i] = 1.f;  // K^ is K<- when R = 0
            } else if (CH) {
                ld8(eR + c0, eR8);
            }
#pragma unroll
            for (int k = 0; k < C / 16; ++k) {
                const int l = l0 + 16 * k, jj = (cg & 7) ^ (l & 7);
                float kv[8], o[8];
                unpack8(*reinterpret_cast<const uint4 *>(sKQ + a * 16384 + l * 128 + jj * 16), kv);
                const float el = CH ? 0.f : __expf(sG[l]);
#pragma unroll
                for (int i = 0; i < 8; ++i) o[i] = kv[i] * (CH ? (fb ? 1.f : eR8[i]) : el);
                *reinterpret_cast<uint4 *>(sKL + a * 8192 + l * 128 + jj * 16) = pack8(o);
            }
        }
    }
    {  // V has landed in Q's place
        const bool okv = mbar_wait_bounded(&bars[0], 1, kSpin, err);
        if (!__syncthreads_and(okv)) goto cleanup;
    }
    if (DEC) {  // the write gate: V <- w . V (zero beyond the sequence end)
        const int cg = tid & 15, c0 = cg * 8, a = cg >> 3, l0 = tid >> 4;
#pragma unroll
        for (int k = 0; k < C / 16; ++k) {
            const int l = l0 + 16 * k, j = (cg & 7) ^ (l & 7);
            float w8[8], vv[8];
            if (l < len) {
                ld8(wg + ((size_t)(tstart + l) * geo.H + h) * D + c0, w8);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) w8[i] = 0.f;
            }
            uint4 *vp = reinterpret_cast<uint4 *>(sV + a * 16384 + l * 128 + j * 16);
            unpack8(*vp, vv);
#pragma unroll
            for (int i = 0; i < 8; ++i) vv[i] *= w8[i];
            *vp = pack8(vv);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // U^T = V^T T^T -> TMEM[0:64), W<-^T = K<-^T T^T -> TMEM[64:128)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, 64, 1, 0);
        const uint64_t bd = sdesc_sw128(smem_u32(sT), 16, 1024);
        const uint64_t av = sdesc_sw128(smem_u32(sV), 16384, 1024);
        const uint64_t ak = sdesc_sw128(smem_u32(sKL), 8192, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            mma_bf16_ss(tmem, sdesc_add(av, kk * 2048), sdesc_add(bd, kk * 32), id, kk > 0);
            mma_bf16_ss(tmem + 64, sdesc_add(ak, kk * 2048), sdesc_add(bd, kk * 32), id, kk > 0);
        }
        mma_commit(&bars[1]);
    }
    {
        // the second commit on this barrier, or the first on the exact route
        const bool ok = mbar_wait_bounded(&bars[1], fb ? 0 : 1, kSpin, err);
        if (!__syncthreads_and(ok)) goto cleanup;  // V and K<- are no longer read
    }
    tc_fence_after();
    {
        // U^T as [d][token] (this thread: row d, 32 tokens) -> staging in the
        // K/Q area (128-byte swizzle) -> TMA store; W<- (this thread: column d)
        const int d = qd * 32 + lane;
        float u[32], w[32];
        tmem_ld16(tmem + lb + hf * 32, u);
        tmem_ld16(tmem + lb + hf * 32 + 16, u + 16);
        tmem_ld16(tmem + lb + 64 + hf * 32, w);
        tmem_ld16(tmem + lb + 64 + hf * 32 + 16, w + 16);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int j = hf * 4 + jj;
            const uint32_t off = d * 128 + ((j ^ (d & 7)) << 4);
            *reinterpret_cast<uint4 *>(sKQ + off) = pack8(u + jj * 8);
        }
        // W<- goes straight to the workspace in token-major order: per token,
        // a warp writes 32 consecutive features (64 contiguous bytes)
        __nv_bfloat16 *wg = ws.W + slot * (C * D) + d;
#pragma unroll
        for (int i = 0; i < 32; ++i) wg[(hf * 32 + i) * D] = __float2bfloat16_rn(w[i]);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        tma_store_2d(&tm_Ust, sKQ, 0, (int)(slot * D));
        bulk_commit_group();
    }
cleanup:
    // shared memory must outlive the stores' reads
    if (tid == 0 || tid == kWyTmaThread) bulk_wait_group_read<0>();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kWyTmemCols);
}

// ------------------------------------------------------------------ state kernel
// Warp roles (13 warps):
//   warps 0-7   state chain: S epilogue and Z epilogue.  Warp w serves TMEM
//               lane quadrant (w & 3) -- state rows d = 32 (w & 3) + lane -- and
//               column half (w >> 2) of the accumulators it touches.
//   warps 8-11  output: O^T (TMEM) -> shared staging -> TMA store.
//   warp 12     MMA issue: every tcgen05.mma, in chunk order, never waiting on
//               a load slot, so it answers the chain's hand-offs at once.
//   warp 13     TMA: loads chunk r + 2 into a stage once chunk r's MMAs are done.
// The roles hand over through mbarriers only; the chain never waits on the
// output path.  TMEM columns: S [0,128); two buffers [Z^T | O^T] at [128,256)
// and [256,384), filled by one N = 128 MMA per k-step; and the bf16 A
// operands of the MMAs -- S [384,448) and Z^T [448,480), two elements per
// column -- so the MMAs read only B from shared memory.
struct StSmem {
    // per stage: [W<-; Q<-] stacked along N (128 x 128, K-major B: each 64-column
    // atom holds W<- rows then Q<- rows),
    // K-> (64 x 128, MN-major B), U^T (128 x 64), A (64 x 64, K-major B)
    static constexpr uint32_t WQ = 0, K = 32768, UT = 49152, A = 65536;
    static constexpr uint32_t STAGE = 73728;
    static constexpr uint32_t DEC = 2 * STAGE;      // decay rows [2][up to 4][128] fp32
    static constexpr uint32_t OST = DEC + 4096;     // O staging for the TMA store [64][128]
    static constexpr uint32_t BARS = OST + 16384;
    static constexpr uint32_t TOTAL = BARS + 256;
    // bytes one stage's loads deliver, with nd decay rows
    static constexpr uint32_t tx(int nd) { return 4 * kTileBytes + kHalfBytes + nd * kDecBytes; }
};
constexpr int kChainThreads = 256, kOutThreads = 128;
constexpr int kStThreads = kChainThreads + kOutThreads + 64;
constexpr uint32_t kStTmemCols = 512;

__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int n) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Named barrier that also ANDs a predicate over its n threads, so that a
// decision taken after a bounded wait is the same in every thread of a role.
__device__ __forceinline__ bool named_sync_and(int id, int n, bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
// Chain -> MMA-warp hand-offs on hardware named barriers (the chain warps
// arrive, the MMA warp syncs).  Both sides pass each barrier exactly twice per
// chain step on every path, error paths included, so neither can be left
// waiting.
//
// SUB (the method's chunk, 64 or 16): a stage holds one 64-token tile; with
// 16-token chunks the chain takes four steps per stage.  Step j uses rows
// 16j.. of the tile: [Z_j^T | O_j^T] = S [W<-_j; Q<-_j]^T (N = 32, the -W<- and
// Q<- rows loaded as alternating 16-row blocks so that each step's pair is
// contiguous), S <- S Diag(decay_j) + Z_j^T K->_j and O_j^T += Z_j^T A_jj^T
// with the diagonal 16 x 16 block of A; the TMEM buffer holds
// [Z_0 O_0 Z_1 O_1 ...] in 16-column blocks.
constexpr int kBarOpsS = 2, kBarOpsZ = 3;
constexpr int kOpsThreads = 256 + 32;

template <int SUB>
__global__ void __launch_bounds__(kStThreads, 1)
state_kernel(const __grid_constant__ CUtensorMap tm_W, const __grid_constant__ CUtensorMap tm_U,
             const __grid_constant__ CUtensorMap tm_Q, const __grid_constant__ CUtensorMap tm_K,
             const __grid_constant__ CUtensorMap tm_A, const __grid_constant__ CUtensorMap tm_out,
             const float *__restrict__ S0, __nv_bfloat16 *__restrict__ out,
             float *__restrict__ S_final, const int32_t *__restrict__ cu, Geo geo, Ws ws,
             unsigned int *err) {
    static_assert(SUB == C || SUB == 16, "method chunk of 64 or 16 tokens");
    constexpr int NSUB = C / SUB;  // chain steps per stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + StSmem::BARS);  // [2] TMA stage loaded
    uint64_t *barZ = full + 4;   // mma: Z^T accumulated
    uint64_t *barS = full + 5;   // mma: S update accumulated
    uint64_t *barO = full + 6;   // [2] mma: O^T buffer complete
    uint64_t *oFree = full + 8;  // [2] output warps: O^T buffer read (one arrival per warp)
    uint32_t *tslot = reinterpret_cast<uint32_t *>(full + 10);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x;
    const int s = geo.varlen ? ws.order[unit / geo.H] : unit / geo.H;
    const int h = unit % geo.H;
    long t0, t1;
    seq_bounds(cu, s, geo.T, geo.T_total, t0, t1);
    const int gc0 = geo.varlen ? ws.chunk_start[s] : s * geo.nc;
    const int nch = (int)((t1 - t0 + C - 1) / C);
    if (kChecked) {  // checked build: the sequence's tokens and the slots of its chunks
        const long long rows = geo.varlen ? (long long)geo.T_total : (long long)geo.B * geo.T;
        const long long nsl = (long long)geo.n_slots * geo.H;
        const long long sl0 = (long long)gc0 * geo.H + h, sl1 = (long long)(gc0 + nch - 1) * geo.H + h;
        if (!(chk_span(s, 1, geo.n_seq, err) && chk_span(t0, t1 - t0, rows, err) &&
              (nch == 0 || (chk_span(sl0, 1, nsl, err) && chk_span(sl1, 1, nsl, err))) &&
              chk_tma(h * D, 0, 2, (long long)geo.H * D, 1, err)))
            return;  // whole CTA, before any sync
    }

    // stage r & 1 <- chunk r's operands and decay rows; -W<- and Q<- arrive as
    // alternating SUB-row blocks (their maps have SUB-row boxes)
    auto issue = [&](int r) {
        uint8_t *st = sm + (r & 1) * StSmem::STAGE;
        uint64_t *bar = &full[r & 1];
        const size_t sl = (size_t)(gc0 + r) * geo.H + h;
        mbar_arrive_expect_tx(bar, StSmem::tx(NSUB));
#pragma unroll
        for (int b = 0; b < NSUB; ++b) {
            const int y = (int)(sl * C) + b * SUB;
            tma_load_2d(st + StSmem::WQ + 2 * b * SUB * 128, &tm_W, bar, 0, y);
            tma_load_2d(st + StSmem::WQ + 16384 + 2 * b * SUB * 128, &tm_W, bar, 64, y);
            tma_load_2d(st + StSmem::WQ + (2 * b + 1) * SUB * 128, &tm_Q, bar, 0, y);
            tma_load_2d(st + StSmem::WQ + 16384 + (2 * b + 1) * SUB * 128, &tm_Q, bar, 64, y);
        }
        tma_load_2d(st + StSmem::UT, &tm_U, bar, 0, (int)(sl * D));
        tma_load_2d(st + StSmem::K, &tm_K, bar, 0, (int)(sl * C));
        tma_load_2d(st + StSmem::K + 8192, &tm_K, bar, 64, (int)(sl * C));
        tma_load_2d(st + StSmem::A, &tm_A, bar, 0, (int)(sl * C));
        bulk_load(sm + StSmem::DEC + (r & 1) * NSUB * kDecBytes, ws.dec + sl * NSUB * D,
                  NSUB * kDecBytes, bar);
    };
    // The TMA thread initialises the stage barriers and issues the first two
    // stages before the CTA barrier, overlapping the TMEM allocation and the
    // S0 load.
    constexpr int kStTmaThread = 13 * 32;
    if (tid == kStTmaThread) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        fence_mbar_init();
        if (nch > 0) {
            prefetch_tmap(&tm_W);
            prefetch_tmap(&tm_U);
            prefetch_tmap(&tm_Q);
            prefetch_tmap(&tm_K);
            prefetch_tmap(&tm_A);
            prefetch_tmap(&tm_out);
            issue(0);
            if (nch > 1) issue(1);
        }
    }
    if (tid == 0) {
        mbar_init(barZ, 1);
        mbar_init(barS, 1);
        mbar_init(&barO[0], 1);
        mbar_init(&barO[1], 1);
        mbar_init(&oFree[0], kOutThreads / 32);
        mbar_init(&oFree[1], kOutThreads / 32);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, kStTmemCols);
        tmem_relinquish();
    }
    // the chain warps' rows of S0 (or 0), loaded before the barrier as well
    float s0v[64];
    if (warp < 8) {
        const int d = (warp & 3) * 32 + lane;
        const size_t soff = ((size_t)s * geo.H + h) * (size_t)D * D + (size_t)d * D + (warp >> 2) * 64;
#pragma unroll
        for (int i4 = 0; i4 < 16; ++i4) {  // 16-byte loads (S0 rows are 16-byte aligned)
            const float4 t = S0 ? reinterpret_cast<const float4 *>(S0 + soff)[i4]
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            s0v[4 * i4] = t.x; s0v[4 * i4 + 1] = t.y; s0v[4 * i4 + 2] = t.z; s0v[4 * i4 + 3] = t.w;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t tS = tmem, tZO0 = tmem + 128, tS16 = tmem + 384, tZ16 = tmem + 448;
    bool ok = true;

    if (warp < 8) {
        // ===================== state chain =====================
        const int qd = warp & 3, hf = warp >> 2;
        const int d = qd * 32 + lane;
        const uint32_t lb = (uint32_t)(qd * 32) << 16;
        const size_t soff = ((size_t)s * geo.H + h) * (size_t)D * D + (size_t)d * D + hf * 64;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) tmem_st16(tS + lb + hf * 64 + cb * 16, s0v + cb * 16);  // S <- S0
        tmem_wait_st();
        for (int r = 0; r < nch; ++r) {
            const uint8_t *st = sm + (r & 1) * StSmem::STAGE;
            if (ok) ok = mbar_wait_bounded(&full[r & 1], (r >> 1) & 1, kSpin, err);
            for (int j = 0; j < NSUB; ++j) {
            const int q = r * NSUB + j;  // chain step
            if (ok && q > 0) ok = mbar_wait_bounded(barS, (q - 1) & 1, kSpin, err);
            ok = __all_sync(0xffffffffu, ok);  // the TMEM accesses below are warp-wide
            float v[64];
            if (ok) {  // S (fp32) -> bf16 operand in TMEM
                tc_fence_after();
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) tmem_ld16(tS + lb + hf * 64 + cb * 16, v + cb * 16);
                tmem_wait_ld();
                float p[32];  // bf16 pairs
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 w = pack8(v + i * 8);
                    p[4 * i] = __uint_as_float(w.x);
                    p[4 * i + 1] = __uint_as_float(w.y);
                    p[4 * i + 2] = __uint_as_float(w.z);
                    p[4 * i + 3] = __uint_as_float(w.w);
                }
                tmem_st16(tS16 + lb + hf * 32, p);
                tmem_st16(tS16 + lb + hf * 32 + 16, p + 16);
                tmem_wait_st();
                tc_fence_before();
            }
            // the Z and O MMAs need only the bf16 copy: release it first
            named_arrive(kBarOpsS, kOpsThreads);
            if (ok) {  // S <- S Diag(decay), needed by the S-update MMA (after opsZ)
                const float *dec = reinterpret_cast<const float *>(sm + StSmem::DEC) +
                                   ((r & 1) * NSUB + j) * D + hf * 64;
#pragma unroll
                for (int i = 0; i < 64; ++i) v[i] *= dec[i];
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) tmem_st16(tS + lb + hf * 64 + cb * 16, v + cb * 16);
                tmem_wait_st();
            }
            if (ok) ok = mbar_wait_bounded(barZ, q & 1, kSpin, err);
            ok = __all_sync(0xffffffffu, ok);
            if (ok && SUB == C) {  // Z^T = U^T - S W<-^T -> bf16 A operand in TMEM (this thread: 32 tokens)
                tc_fence_after();
                float z[32];
                const uint32_t tZ = tZO0 + (r & 1) * 128;
                tmem_ld16(tZ + lb + hf * 32, z);
                tmem_ld16(tZ + lb + hf * 32 + 16, z + 16);
                tmem_wait_ld();
                const uint8_t *urow = st + StSmem::UT + d * 128;
                float p[16];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int c16 = hf * 4 + jj;
                    float u[8];
                    unpack8(*reinterpret_cast<const uint4 *>(urow + ((c16 ^ (d & 7)) << 4)), u);
#pragma unroll
                    for (int i = 0; i < 8; ++i) u[i] -= z[jj * 8 + i];
                    const uint4 w = pack8(u);
                    p[4 * jj] = __uint_as_float(w.x);
                    p[4 * jj + 1] = __uint_as_float(w.y);
                    p[4 * jj + 2] = __uint_as_float(w.z);
                    p[4 * jj + 3] = __uint_as_float(w.w);
                }
                tmem_st16(tZ16 + lb + hf * 16, p);
                tmem_wait_st();
                tc_fence_before();
            } else if (ok) {  // 16-token chunk j: this thread 8 of its tokens
                tc_fence_after();
                float z[8];
                tmem_ld8(tZO0 + (r & 1) * 128 + 32 * j + hf * 8 + lb, z);
                tmem_wait_ld();
                const uint8_t *urow = st + StSmem::UT + d * 128;
                float u[8];
                unpack8(*reinterpret_cast<const uint4 *>(urow + (((2 * j + hf) ^ (d & 7)) << 4)), u);
#pragma unroll
                for (int i = 0; i < 8; ++i) u[i] -= z[i];
                const uint4 w = pack8(u);
                const float p[4] = {__uint_as_float(w.x), __uint_as_float(w.y),
                                    __uint_as_float(w.z), __uint_as_float(w.w)};
                tmem_st4(tZ16 + lb + hf * 4, p);
                tmem_wait_st();
                tc_fence_before();
            }
            named_arrive(kBarOpsZ, kOpsThreads);
            }  // chain steps
        }
        if (ok && nch > 0) ok = mbar_wait_bounded(barS, (nch * NSUB - 1) & 1, kSpin, err);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (ok && S_final) {
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float v[16];
                tmem_ld16(tS + lb + hf * 64 + cb * 16, v);
                tmem_wait_ld();
                float4 *dst = reinterpret_cast<float4 *>(S_final + soff + cb * 16);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        }
    } else if (warp < 12) {
        // ===================== output =====================
        const int qd = warp & 3;
        const int d = qd * 32 + lane;
        const int otid = tid - kChainThreads;
        const uint32_t lb = (uint32_t)(qd * 32) << 16;
        __nv_bfloat16 *ost = reinterpret_cast<__nv_bfloat16 *>(sm + StSmem::OST);
        for (int r = 0; r < nch; ++r) {
            // every output thread goes on, or all stop: the named barriers
            // below need all of them
            ok = named_sync_and(1, kOutThreads,
                                mbar_wait_bounded(&barO[r & 1], (r >> 1) & 1, kSpin, err));
            if (!ok) break;
            tc_fence_after();
            float o[64];  // token order: O sits after Z in each SUB-column block
#pragma unroll
            for (int cb = 0; cb < 4; ++cb)
                tmem_ld16(tZO0 + (r & 1) * 128 + (SUB == C ? 64 + cb * 16 : 32 * cb + 16) + lb,
                          o + cb * 16);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&oFree[r & 1]);
            const long ts = t0 + (long)r * C;
            const int len = (int)min((long)C, t1 - ts);
            const int kp = geo.keep;
            if (kp > 1 && len == C && C % kp == 0 && ts % kp == 0) {
                // the last substep of each token: C / kp rows staged, one TMA store
                if (otid == 0) bulk_wait_group_read<0>();  // staging buffer free again
                named_sync(1, kOutThreads);
                if (kp == 2) {
#pragma unroll
                    for (int m = 0; m < 32; ++m) ost[m * D + d] = __float2bfloat16_rn(o[2 * m + 1]);
                } else if (kp == 4) {
#pragma unroll
                    for (int m = 0; m < 16; ++m) ost[m * D + d] = __float2bfloat16_rn(o[4 * m + 3]);
                } else {
                    int j = 0, m = 0;
#pragma unroll
                    for (int i = 0; i < 64; ++i) {
                        if (j == kp - 1) {
                            ost[m * D + d] = __float2bfloat16_rn(o[i]);
                            ++m;
                        }
                        if (++j == kp) j = 0;
                    }
                }
                fence_proxy_async_smem();
                named_sync(1, kOutThreads);
                if (otid == 0) {
                    tma_store_2d(&tm_out, ost, h * D, (int)(ts / kp));
                    bulk_commit_group();
                }
            } else if (kp > 1) {  // partial chunk, or kp not dividing C: plain stores
                int j = (int)(ts % kp);
                long t = ts / kp;
                __nv_bfloat16 *og = out + (size_t)h * D + d;
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    if (i < len && j == kp - 1) og[(size_t)t * geo.H * D] = __float2bfloat16_rn(o[i]);
                    if (++j == kp) {
                        j = 0;
                        ++t;
                    }
                }
            } else if (len == C) {
                if (otid == 0) bulk_wait_group_read<0>();  // staging buffer free again
                named_sync(1, kOutThreads);
#pragma unroll
                for (int i = 0; i < 64; ++i) ost[i * D + d] = __float2bfloat16_rn(o[i]);
                fence_proxy_async_smem();
                named_sync(1, kOutThreads);
                if (otid == 0) {
                    tma_store_2d(&tm_out, ost, h * D, (int)ts);
                    bulk_commit_group();
                }
            } else {
                __nv_bfloat16 *og = out + ((size_t)ts * geo.H + h) * D + d;
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if (i < len) og[(size_t)i * geo.H * D] = __float2bfloat16_rn(o[i]);
            }
        }
        if (otid == 0) bulk_wait_group_read<0>();
    } else if (tid == kStTmaThread) {
        // ===================== TMA loads (stages 0 and 1 are in flight) =====================
        int issued = nch < 2 ? nch : 2;
        // stage r & 1 is free once chunk r - 2's MMAs (the last is O2) are done
        for (int r = 2; r < nch && ok; ++r) {
            ok = mbar_wait_bounded(&barO[r & 1], ((r - 2) >> 1) & 1, kSpin, err);
            if (!ok) break;
            issue(r);
            issued = r + 1;
        }
        // let every load this thread issued land before the CTA can exit
        for (int i = issued - 2; i < issued; ++i)
            if (i >= 0) mbar_wait_bounded(&full[i & 1], (i >> 1) & 1, kSpin, err);
    } else if (warp == 12) {
        // ===================== MMA issue (lane 0; the warp syncs) =====================
        const uint32_t idZO = idesc_bf16(128, 2 * SUB, 0, 0);
        const uint32_t idO = idesc_bf16(128, SUB, 0, 0);
        const uint32_t idS = idesc_bf16(128, 128, 0, 1);
        // operand descriptors, built once; k-steps only advance the start address
        const uint64_t dWQ0 = sdesc_sw128(smem_u32(sm + StSmem::WQ), 16, 1024);
        const uint64_t dK0 = sdesc_sw128(smem_u32(sm + StSmem::K), 8192, 1024);
        const uint64_t dA0 = sdesc_sw128(smem_u32(sm + StSmem::A), 16, 1024);
        const uint32_t stage16 = StSmem::STAGE >> 4;  // stage stride in descriptor units
        for (int r = 0; r < nch; ++r) {
            const uint32_t tZr = tZO0 + (r & 1) * 128;
            const uint64_t so = (r & 1) ? stage16 : 0;
            const uint64_t dwq = dWQ0 + so, dk = dK0 + so, da = dA0 + so;
            // this buffer's O half must have been read out (chunk r - 2)
            if (ok && lane == 0 && r >= 2)
                ok = mbar_wait_bounded(&oFree[r & 1], ((r - 2) >> 1) & 1, kSpin, err);
            for (int j = 0; j < NSUB; ++j) {
                __syncwarp();
                // the chain has written S in bf16 (and so has seen chunk r's stage land)
                named_sync(kBarOpsS, kOpsThreads);
                const uint32_t tZj = tZr + 2 * SUB * j;  // [Z_j | O_j]
                if (ok && lane == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // [Z_j^T | O_j^T] = S [W<-_j; Q<-_j]^T
                        mma_bf16_ts(tZj, tS16 + kk * 8,
                                    sdesc_add(dwq, 2 * SUB * j * 128 + (kk >> 2) * 16384 +
                                                       (kk & 3) * 32),
                                    idZO, kk > 0);
                    mma_commit(barZ);
                }
                __syncwarp();
                named_sync(kBarOpsZ, kOpsThreads);
                if (ok && lane == 0) {
                    tc_fence_after();
                    constexpr int KS = SUB / 16;  // k-steps over the chunk's tokens
#pragma unroll
                    for (int kk = 0; kk < KS; ++kk)  // S += Z_j^T K->_j
                        mma_bf16_ts(tS, tZ16 + kk * 8, sdesc_add(dk, (j * KS + kk) * 2048), idS, 1);
                    mma_commit(barS);
#pragma unroll
                    for (int kk = 0; kk < KS; ++kk)  // O_j^T += Z_j^T A_jj^T
                        mma_bf16_ts(tZj + SUB, tZ16 + kk * 8,
                                    sdesc_add(da, j * SUB * 128 + (j * KS + kk) * 32), idO, 1);
                    if (j == NSUB - 1) mma_commit(&barO[r & 1]);
                }
            }
        }
    }
    // every role ends here; the chain and output roles have waited for the
    // last MMAs, so TMEM can be released
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kStTmemCols);
}

}  // namespace tc
}  // namespace gdr

// ====================================================================== host side
using namespace gdr;
using namespace gdr::tc;

namespace {

struct WsLayout {
    size_t plan, dec, W, U, Q, K, A, total;
    int n_slots;
};

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// nsub: decay rows per tile (one per method chunk: 1 at 64 tokens, 4 at 16)
WsLayout ws_layout(int B, int T, int H, int n_seq, int varlen, int nsub = 1) {
    WsLayout L;
    L.n_slots = varlen ? (T + C - 1) / C + n_seq : B * ((T + C - 1) / C);
    const size_t tiles = (size_t)L.n_slots * H;
    size_t o = 0;
    L.plan = o; o += up256(sizeof(int) * (size_t)(2 * (varlen ? n_seq : 0) + 1));
    L.dec = o;  o += up256(tiles * nsub * D * 4);
    L.W = o;    o += up256(tiles * C * D * 2);
    L.U = o;    o += up256(tiles * C * D * 2);
    L.Q = o;    o += up256(tiles * C * D * 2);
    L.K = o;    o += up256(tiles * C * D * 2);
    L.A = o;    o += up256(tiles * C * C * 2);
    L.total = o;
    return L;
}

using namespace gdr_host::tmap;

// Spread limit of the factorised Gram weights (Geo::spread_limit).
std::atomic<float> g_spread_limit{60.f};
constexpr float kSpreadLimitMax = 80.f;  // e^80 and e^-80 stay normal fp32 / bf16

size_t wy_smem_bytes(bool ch) {  // + 1024 for the in-kernel alignment
    return 1024 + WySmem::small(ch) + WySmem::small_bytes(ch);
}

}  // namespace

namespace gdr_host {

bool tc_applies(int dk, int dv, int chunk, gdr_dtype dtype) {
    return dtype == GDR_BF16 && dk == D && dv == D && chunk == C;
}

// The prefill entry points also run 16-token chunks on the tensor cores
// (gdr_fwd_noalloc keeps to 64)
bool tc_applies_fwd(int dk, int dv, int chunk, gdr_dtype dtype, gdr_gate, int) {
    return dtype == GDR_BF16 && dk == D && dv == D && (chunk == C || chunk == 16);
}

size_t tc_workspace_bytes(int B, int T, int H, int n_seq, int varlen, gdr_gate) {
    return ws_layout(B, T, H, n_seq, varlen).total;
}

size_t tc_workspace_bytes_chunk(int B, int T, int H, int n_seq, int varlen, gdr_gate,
                                int chunk) {
    return ws_layout(B, T, H, n_seq, varlen, chunk == 16 ? C / 16 : 1).total;
}

size_t tc_workspace_bytes_gdn2_chunk(int B, int T, int H, int n_seq, int varlen, int chunk) {
    return ws_layout(B, T, H, n_seq, varlen, chunk == 16 ? C / 16 : 1).total;
}

static cudaError_t tc_dispatch(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *eg, const float *wg,
                               const float *S0, void *out, float *S_final, int B, int T, int H,
                               const int32_t *cu, int n_seq, gdr_gate gate, void *workspace,
                               size_t ws_bytes, unsigned int *err, cudaStream_t st,
                               int keep = 1, int chunk = C) {
    const int varlen = cu != nullptr;
    const bool c16 = chunk == 16;
    if (!(chunk == C || c16)) return cudaErrorInvalidValue;
    const int sub = c16 ? 16 : C;
    const WsLayout L = ws_layout(B, T, H, n_seq, varlen, C / sub);
    if (ws_bytes < L.total || !err) return cudaErrorInvalidValue;
    uint8_t *wsb = (uint8_t *)workspace;
    Ws ws;
    ws.chunk_start = (int *)(wsb + L.plan);
    ws.order = ws.chunk_start + (n_seq + 1);
    ws.dec = (float *)(wsb + L.dec);
    ws.W = (__nv_bfloat16 *)(wsb + L.W);
    ws.U = (__nv_bfloat16 *)(wsb + L.U);
    ws.Q = (__nv_bfloat16 *)(wsb + L.Q);
    ws.K = (__nv_bfloat16 *)(wsb + L.K);
    ws.A = (__nv_bfloat16 *)(wsb + L.A);
    Geo geo;
    geo.B = B; geo.T = T; geo.H = H; geo.n_seq = varlen ? n_seq : B;
    geo.nc = (T + C - 1) / C; geo.varlen = varlen; geo.T_total = B * T; geo.n_slots = L.n_slots;
    geo.keep = keep;
    geo.spread_limit = g_spread_limit.load(std::memory_order_relaxed);

    const size_t tiles = (size_t)L.n_slots * H;
    if (tiles * D >= ((size_t)1 << 31)) return cudaErrorInvalidValue;  // 32-bit TMA rows
    const uint64_t tok_rows = (uint64_t)B * T;
    const uint64_t HD = (uint64_t)H * D;
    CUtensorMap mq, mk, mv, mg, mW, mU, mQ, mK, mA, mo;
    memset(&mg, 0, sizeof(mg));
    const bool have_tokens = tok_rows > 0;
    if (have_tokens) {
        if (!make_map(&mq, kBF, q, HD, tok_rows, HD * 2, 64, 64, kSW) ||
            !make_map(&mk, kBF, k, HD, tok_rows, HD * 2, 64, 64, kSW) ||
            !make_map(&mv, kBF, v, HD, tok_rows, HD * 2, 64, 64, kSW) ||
            (gate == GDR_GATE_PER_KEY_CHANNEL &&
             !make_map(&mg, kF32, g, HD, tok_rows, HD * 4, D, 64, kNoSW)) ||
            !make_map(&mW, kBF, ws.W, D, tiles * C, D * 2, 64, sub, kSW) ||
            !make_map(&mU, kBF, ws.U, C, tiles * D, C * 2, 64, 128, kSW) ||
            !make_map(&mQ, kBF, ws.Q, D, tiles * C, D * 2, 64, sub, kSW) ||
            !make_map(&mK, kBF, ws.K, D, tiles * C, D * 2, 64, 64, kSW) ||
            !make_map(&mA, kBF, ws.A, C, tiles * C, C * 2, 64, 64, kSW) ||
            !make_map(&mo, kBF, out, HD, tok_rows / keep, HD * 2, D,
                      C % keep == 0 ? C / keep : 64, kNoSW))
            return cudaErrorInvalidValue;
    } else {
        memset(&mW, 0, sizeof(mW));
        mq = mk = mv = mU = mQ = mK = mA = mo = mW;
    }
    cudaError_t e;
    if (varlen) {
        ProfToken tk = prof_begin(GDR_K_TC_PLAN, st);
        plan_kernel<<<1, 256, 0, st>>>(cu, n_seq, B * T, ws.chunk_start, ws.order);
        prof_end(tk, st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const bool ch = gate == GDR_GATE_PER_KEY_CHANNEL;
    if (have_tokens && L.n_slots > 0) {
        const bool dec = eg != nullptr;
        // decoupled gates run the per-channel kernel; a scalar decay is broadcast
        const size_t smem = wy_smem_bytes(ch || dec);
        auto kern = dec ? (ch ? (c16 ? wy_kernel<true, true, false, 16> : wy_kernel<true, true>)
                              : (c16 ? wy_kernel<true, true, true, 16> : wy_kernel<true, true, true>))
                        : ch ? (c16 ? wy_kernel<true, false, false, 16> : wy_kernel<true>)
                             : c16 ? wy_kernel<false, false, false, 16>
                                   : wy_kernel<false>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        dim3 grid((unsigned)L.n_slots, (unsigned)H);
        ProfToken tk = prof_begin(GDR_K_TC_WY, st);
        kern<<<grid, kWyThreads, smem, st>>>(mq, mk, mv, mg, mU, mA, g, beta, eg, wg, cu, geo, ws,
                                             err);
        prof_end(tk, st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        const size_t smem = 1024 + StSmem::TOTAL;
        auto skern = c16 ? state_kernel<16> : state_kernel<C>;
        if ((e = cudaFuncSetAttribute(skern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        ProfToken tk = prof_begin(GDR_K_TC_STATE, st);
        skern<<<(unsigned)(geo.n_seq * H), kStThreads, smem, st>>>(
            mW, mU, mQ, mK, mA, mo, S0, (__nv_bfloat16 *)out, S_final, cu, geo, ws, err);
        prof_end(tk, st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t fwd_tc_dispatch(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *S0, void *out, float *S_final, int B,
                            int T, int H, const int32_t *cu, int n_seq, gdr_gate gate,
                            void *workspace, size_t ws_bytes, unsigned int *err,
                            cudaStream_t st, int chunk) {
    return tc_dispatch(q, k, v, g, beta, nullptr, nullptr, S0, out, S_final, B, T, H, cu, n_seq,
                       gate, workspace, ws_bytes, err, st, 1, chunk);
}

// Gated DeltaProduct: the prefill over the virtual sequence of keep substeps
// per token (T virtual rows per sequence), out [B, T / keep, H, d_v] receiving
// the last substep of each token.
cudaError_t fwd_tc_keep_dispatch(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *S0, void *out, float *S_final,
                                 int B, int T, int H, const int32_t *cu, int n_seq, gdr_gate gate,
                                 int keep, void *workspace, size_t ws_bytes, unsigned int *err,
                                 cudaStream_t st, int chunk) {
    if (keep < 1 || T % keep) return cudaErrorInvalidValue;
    return tc_dispatch(q, k, v, g, beta, nullptr, nullptr, S0, out, S_final, B, T, H, cu, n_seq,
                       gate, workspace, ws_bytes, err, st, keep, chunk);
}

// Gated DeltaNet-2: erase gate eg [.., d_k], write gate wg [.., d_v]; the decay
// per key channel or one scalar per token.
cudaError_t fwd_tc_gdn2_dispatch(const void *q, const void *k, const void *v, const float *g,
                                 const float *eg, const float *wg, const float *S0, void *out,
                                 float *S_final, int B, int T, int H, const int32_t *cu, int n_seq,
                                 gdr_gate gate, void *workspace, size_t ws_bytes,
                                 unsigned int *err, cudaStream_t st, int chunk) {
    if (!eg || !wg) return cudaErrorInvalidValue;
    return tc_dispatch(q, k, v, g, nullptr, eg, wg, S0, out, S_final, B, T, H, cu, n_seq, gate,
                       workspace, ws_bytes, err, st, 1, chunk);
}

}  // namespace gdr_host

extern "C" float gdr_set_gram_spread_limit(float limit) {
    float prev = g_spread_limit.load();
    if (limit == limit) {  // NaN leaves the limit as it is
        limit = limit < 0.f ? 0.f : (limit > kSpreadLimitMax ? kSpreadLimitMax : limit);
        prev = g_spread_limit.exchange(limit);
    }
    return prev;
}
