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
// This needs |G_l - G_r| < ~80 per channel inside a chunk (bf16/fp32 range);
// the SIMT path has no such limit.
//
// Tokens of a chunk that runs past the end of its sequence are zeroed in
// shared memory (k = q = v = 0, beta = 0, g = 0), which leaves every valid row
// unchanged.  Every wait on an mbarrier is bounded: on expiry the kernel
// records a timeout in the device error word, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gdr {
namespace tc {

using namespace sm100;

constexpr int C = 64;
constexpr int D = 128;
constexpr int kThreads = 128;
constexpr uint32_t kSpin = 1u << 24;  // poll limit of every mbarrier wait
constexpr uint32_t kTmemCols = 256;

constexpr uint32_t kTileBytes = C * D * 2;   // 16 KB: one [64][128] bf16 tile
constexpr uint32_t kHalfBytes = C * 64 * 2;  // 8 KB: one [64][64] bf16 atom column
constexpr uint32_t kDecBytes = D * 4;

struct Geo {
    int B, T, H, n_seq, nc;  // nc: chunks per sequence (regular batches)
    int varlen, T_total, n_slots;
};

struct Ws {
    int *chunk_start;  // [n_seq + 1] (varlen)
    int *order;        // [n_seq] longest first (varlen)
    float *dec;        // [slots*H][128]
    __nv_bfloat16 *W, *U, *Q, *K;  // [slots*H][64][128]
    __nv_bfloat16 *A;              // [slots*H][64][64]
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return (uint8_t *)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

// bf16x8 <-> float8 helpers (16-byte chunks of a tile)
__device__ __forceinline__ void unpack8(const uint4 &u, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ uint4 pack8(const float *f) {
    uint4 u;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return u;
}

// Locate chunk `gcid` of the packed or regular batch: sequence index, first
// token row and valid length.  Returns false for an unused slot.
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

// ------------------------------------------------------------------ WY kernel
struct WySmem {
    static constexpr uint32_t KQ = 0;                    // [K;Q] raw, 2 atoms x 128 rows
    static constexpr uint32_t V = KQ + 2 * 16384;        // 2 atoms x 64 rows
    static constexpr uint32_t KL = V + 2 * 8192;         // K<- (MMA A operand, MN-major)
    static constexpr uint32_t TT = KL + 2 * 8192;        // T, K-major B operand
    static constexpr uint32_t KH = TT + 8192;            // KDA: [K^;Q^] scaled Gram A
    static constexpr uint32_t KC = KH + 2 * 16384;       // KDA: K-check, Gram B
    static constexpr uint32_t end_tc(bool ch) { return ch ? KC + 2 * 8192 : KH; }
    static constexpr int NST = 68;                       // fp32 row stride of N
};

template <bool CH>
__global__ void __launch_bounds__(kThreads)
wy_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g,
          const float *__restrict__ beta, const int32_t *__restrict__ cu, Geo geo, Ws ws,
          unsigned int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint8_t *sKQ = sm + WySmem::KQ, *sV = sm + WySmem::V, *sKL = sm + WySmem::KL;
    uint8_t *sT = sm + WySmem::TT, *sKH = sm + WySmem::KH, *sKC = sm + WySmem::KC;
    float *sN = reinterpret_cast<float *>(sm + WySmem::end_tc(CH));   // [64][NST]
    float *sG = sN + 64 * WySmem::NST;                                 // CH ? [64][128] : [64]
    float *sB = sG + (CH ? 64 * D : 64);                               // beta [64]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sB + 64);           // [2]
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gcid = blockIdx.x, h = blockIdx.y;
    long tstart;
    int len;
    if (!locate_chunk(geo, cu, ws, gcid, tstart, len)) return;  // whole CTA, before any sync
    const size_t slot = (size_t)gcid * geo.H + h;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    if (tid == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        mbar_arrive_expect_tx(&bars[0], 6 * kHalfBytes);
        const int x0 = h * D, y = (int)tstart;
        tma_load_2d(sKQ, &tm_k, &bars[0], x0, y);
        tma_load_2d(sKQ + 16384, &tm_k, &bars[0], x0 + 64, y);
        tma_load_2d(sKQ + 8192, &tm_q, &bars[0], x0, y);
        tma_load_2d(sKQ + 16384 + 8192, &tm_q, &bars[0], x0 + 64, y);
        tma_load_2d(sV, &tm_v, &bars[0], x0, y);
        tma_load_2d(sV + 8192, &tm_v, &bars[0], x0 + 64, y);
    }
    // gates and beta (zero beyond the sequence end), cumulative log-decay G
    if (CH) {
        for (int e = tid; e < C * D; e += kThreads) {
            const int l = e >> 7, c = e & 127;
            sG[e] = (l < len) ? g[((size_t)(tstart + l) * geo.H + h) * D + c] : 0.f;
        }
    } else if (tid < C) {
        sG[tid] = (tid < len) ? g[(size_t)(tstart + tid) * geo.H + h] : 0.f;
    }
    if (tid < C) sB[tid] = (tid < len) ? beta[(size_t)(tstart + tid) * geo.H + h] : 0.f;
    __syncthreads();
    if (CH) {
        float acc = 0.f;  // thread = channel
        for (int l = 0; l < C; ++l) {
            acc += sG[l * D + tid];
            sG[l * D + tid] = acc;
        }
    } else if (warp == 0) {
        float a = sG[lane], b = sG[lane + 32];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float ya = __shfl_up_sync(0xffffffffu, a, off);
            const float yb = __shfl_up_sync(0xffffffffu, b, off);
            if (lane >= off) {
                a += ya;
                b += yb;
            }
        }
        b += __shfl_sync(0xffffffffu, a, 31);
        sG[lane] = a;
        sG[lane + 32] = b;
    }
    const bool ok_ld = mbar_wait_bounded(&bars[0], 0, kSpin, err);
    if (!__syncthreads_and(ok_ld)) goto cleanup;

    // zero the rows beyond the sequence end (whole 128-byte rows: swizzle-agnostic)
    if (len < C) {
        for (int e = tid; e < (C - len) * 8 * 6; e += kThreads) {
            const int r = len + e / 48, part = e % 48, tile = part >> 3, ch16 = part & 7;
            uint8_t *base = tile < 4 ? sKQ + (tile & 1) * 16384 + (tile >> 1) * 8192
                                     : sV + (tile & 1) * 8192;
            *reinterpret_cast<uint4 *>(base + r * 128 + ch16 * 16) = make_uint4(0, 0, 0, 0);
        }
        __syncthreads();
    }
    // decayed operands: K<- = e^G . k (all gates); KDA also the scaled Gram operands
    for (int e = tid; e < C * 16; e += kThreads) {
        const int l = e >> 4, a = (e >> 3) & 1, j = e & 7;
        const int c0 = a * 64 + ((j ^ (l & 7)) << 3);
        const uint32_t off = a * 16384 + l * 128 + j * 16;
        float kv[8], w[8];
        unpack8(*reinterpret_cast<const uint4 *>(sKQ + off), kv);
        if (CH) {
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = __expf(sG[l * D + c0 + i]);
        } else {
            const float s = __expf(sG[l]);
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = s;
        }
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = kv[i] * w[i];
        *reinterpret_cast<uint4 *>(sKL + a * 8192 + l * 128 + j * 16) = pack8(o);
        if (CH) {
            float qv[8], e1[8], e2[8];
            unpack8(*reinterpret_cast<const uint4 *>(sKQ + off + 8192), qv);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float d = sG[l * D + c0 + i] - sG[31 * D + c0 + i];
                e1[i] = __expf(d);
                e2[i] = __expf(-d);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = kv[i] * e1[i];
            *reinterpret_cast<uint4 *>(sKH + off) = pack8(o);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = qv[i] * e1[i];
            *reinterpret_cast<uint4 *>(sKH + off + 8192) = pack8(o);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = kv[i] * e2[i];
            *reinterpret_cast<uint4 *>(sKC + a * 8192 + l * 128 + j * 16) = pack8(o);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // Gram: TMEM[0:64) = [K;Q] (128 x 128) * Kc^T (64 x 128)^T
    if (tid == 0) {
        tc_fence_after();
        const uint8_t *Ab = CH ? sKH : sKQ;
        const uint8_t *Bb = CH ? sKC : sKQ;
        const uint32_t bstride = CH ? 8192 : 16384;
        const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (kk & 3) * 32;
            const uint64_t ad = sdesc_sw128(smem_u32(Ab + (kk >> 2) * 16384 + koff), 16, 1024);
            const uint64_t bd = sdesc_sw128(smem_u32(Bb + (kk >> 2) * bstride + koff), 16, 1024);
            mma_bf16_ss(tmem, ad, bd, id, kk > 0);
        }
        mma_commit(&bars[1]);
    }
    {
        const bool ok = mbar_wait_bounded(&bars[1], 0, kSpin, err);
        if (!__syncthreads_and(ok)) goto cleanup;
    }
    tc_fence_after();
    {
        // rows 0..63 of the accumulator: K K^T; rows 64..127: Q K^T
        const int l = (warp & 1) * 32 + lane;
        float gr[64];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb)
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + cb * 16, gr + cb * 16);
        tmem_wait_ld();
        const float Gl = CH ? 0.f : sG[l];
        if (warp < 2) {
            const float bl = sB[l];
#pragma unroll
            for (int m = 0; m < 64; ++m) {
                const float w = CH ? 1.f : __expf(Gl - sG[m]);
                sN[l * WySmem::NST + m] = (m < l) ? bl * gr[m] * w : 0.f;
            }
        } else {
            __nv_bfloat16 *Ag = ws.A + slot * (C * C) + (size_t)l * C;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float o[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int m = j * 8 + i;
                    const float w = CH ? 1.f : __expf(Gl - sG[m]);
                    o[i] = (m <= l) ? gr[m] * w : 0.f;
                }
                *reinterpret_cast<uint4 *>(Ag + j * 8) = pack8(o);
            }
        }
    }
    __syncthreads();
    // T: (I + N) T = diag(beta); thread j < 64 solves column j by forward substitution
    if (tid < C) {
        const int j = tid;
        float t[C];
#pragma unroll
        for (int i = 0; i < C; ++i) {
            float acc = 0.f;
            const float4 *row = reinterpret_cast<const float4 *>(sN + i * WySmem::NST);
#pragma unroll
            for (int m4 = 0; m4 < (i + 3) / 4; ++m4) {
                const float4 nv = row[m4];
                if (4 * m4 + 0 < i) acc = fmaf(nv.x, t[4 * m4 + 0], acc);
                if (4 * m4 + 1 < i) acc = fmaf(nv.y, t[4 * m4 + 1], acc);
                if (4 * m4 + 2 < i) acc = fmaf(nv.z, t[4 * m4 + 2], acc);
                if (4 * m4 + 3 < i) acc = fmaf(nv.w, t[4 * m4 + 3], acc);
            }
            t[i] = ((i == j) ? sB[j] : 0.f) - acc;
        }
        // T[i][j] -> K-major SW128 tile (row i, column j)
#pragma unroll
        for (int i = 0; i < C; ++i)
            *reinterpret_cast<__nv_bfloat16 *>(sT + sw128_off(i, j)) = __float2bfloat16_rn(t[i]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // U^T = V^T T^T -> TMEM[64:128), W<-^T = K<-^T T^T -> TMEM[128:192)
    if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, 64, 1, 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_sw128(smem_u32(sT + kk * 32), 16, 1024);
            const uint64_t av = sdesc_sw128(smem_u32(sV + kk * 2048), 8192, 1024);
            const uint64_t ak = sdesc_sw128(smem_u32(sKL + kk * 2048), 8192, 1024);
            mma_bf16_ss(tmem + 64, av, bd, id, kk > 0);
            mma_bf16_ss(tmem + 128, ak, bd, id, kk > 0);
        }
        mma_commit(&bars[1]);
    }
    // meanwhile: Q<- and K-> to the workspace, and the chunk decay
    {
        __nv_bfloat16 *Qg = ws.Q + slot * (C * D), *Kg = ws.K + slot * (C * D);
        for (int e = tid; e < C * 16; e += kThreads) {
            const int l = e >> 4, a = (e >> 3) & 1, j = e & 7;
            const int c0 = a * 64 + ((j ^ (l & 7)) << 3);
            const uint32_t off = a * 16384 + l * 128 + j * 16;
            float kv[8], qv[8], wq[8], wk[8];
            unpack8(*reinterpret_cast<const uint4 *>(sKQ + off), kv);
            unpack8(*reinterpret_cast<const uint4 *>(sKQ + off + 8192), qv);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float Gl = CH ? sG[l * D + c0 + i] : sG[l];
                const float Gc = CH ? sG[(C - 1) * D + c0 + i] : sG[C - 1];
                wq[i] = qv[i] * __expf(Gl);
                wk[i] = kv[i] * __expf(Gc - Gl);
            }
            *reinterpret_cast<uint4 *>(Qg + l * D + c0) = pack8(wq);
            *reinterpret_cast<uint4 *>(Kg + l * D + c0) = pack8(wk);
        }
        ws.dec[slot * D + tid] = __expf(CH ? sG[(C - 1) * D + tid] : sG[C - 1]);
    }
    {
        const bool ok = mbar_wait_bounded(&bars[1], 1, kSpin, err);
        if (!__syncthreads_and(ok)) goto cleanup;
    }
    tc_fence_after();
    {
        // thread = feature row d of U^T / W<-^T; write U[l][d], W[l][d]
        const int d = tid;
        __nv_bfloat16 *Ug = ws.U + slot * (C * D), *Wg = ws.W + slot * (C * D);
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            float u[16], w[16];
            tmem_ld16(tmem + lane_base + 64 + cb * 16, u);
            tmem_ld16(tmem + lane_base + 128 + cb * 16, w);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int l = cb * 16 + i;
                Ug[l * D + d] = __float2bfloat16_rn(u[i]);
                Wg[l * D + d] = __float2bfloat16_rn(w[i]);
            }
        }
    }
cleanup:
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ state kernel
struct StSmem {
    // per stage: W, Q, K, U (16 KB each, 2 atom columns of 8 KB), A (8 KB), decay (512 B)
    static constexpr uint32_t W = 0, Q = 16384, K = 32768, U = 49152, A = 65536, DEC = 73728;
    static constexpr uint32_t STAGE = 74752;  // 73 KB, multiple of 1024
    static constexpr uint32_t S = 2 * STAGE;  // bf16 S, 2 atom columns x 128 rows
    static constexpr uint32_t ZT = S + 32768; // bf16 Z^T, 128 rows x 64
    static constexpr uint32_t BARS = ZT + 16384;
    static constexpr uint32_t TOTAL = BARS + 64;
    static constexpr uint32_t TX = 4 * kTileBytes + kHalfBytes + kDecBytes;
};

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
state_kernel(const __grid_constant__ CUtensorMap tm_W, const __grid_constant__ CUtensorMap tm_U,
             const __grid_constant__ CUtensorMap tm_Q, const __grid_constant__ CUtensorMap tm_K,
             const __grid_constant__ CUtensorMap tm_A, const float *__restrict__ S0,
             __nv_bfloat16 *__restrict__ out, float *__restrict__ S_final,
             const int32_t *__restrict__ cu, Geo geo, Ws ws, unsigned int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + StSmem::BARS);  // full[2], mma
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + 3);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int unit = blockIdx.x;
    const int s = geo.varlen ? ws.order[unit / geo.H] : unit / geo.H;
    const int h = unit % geo.H;
    long t0, t1;
    seq_bounds(cu, s, geo.T, geo.T_total, t0, t1);
    const int gc0 = geo.varlen ? ws.chunk_start[s] : s * geo.nc;
    const int nch = (int)((t1 - t0 + C - 1) / C);
    const int d = tid;  // state row owned by this thread (TMEM lane)
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const size_t soff = ((size_t)s * geo.H + h) * (size_t)D * D + (size_t)d * D;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init(&bars[2], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t tS = tmem, tZ = tmem + 128, tO = tmem + 192;

    auto issue = [&](int r) {
        uint8_t *st = sm + (r & 1) * StSmem::STAGE;
        uint64_t *bar = &bars[r & 1];
        const size_t sl = (size_t)(gc0 + r) * geo.H + h;
        const int y = (int)(sl * C);
        mbar_arrive_expect_tx(bar, StSmem::TX);
        tma_load_2d(st + StSmem::W, &tm_W, bar, 0, y);
        tma_load_2d(st + StSmem::W + 8192, &tm_W, bar, 64, y);
        tma_load_2d(st + StSmem::Q, &tm_Q, bar, 0, y);
        tma_load_2d(st + StSmem::Q + 8192, &tm_Q, bar, 64, y);
        tma_load_2d(st + StSmem::K, &tm_K, bar, 0, y);
        tma_load_2d(st + StSmem::K + 8192, &tm_K, bar, 64, y);
        tma_load_2d(st + StSmem::U, &tm_U, bar, 0, y);
        tma_load_2d(st + StSmem::U + 8192, &tm_U, bar, 64, y);
        tma_load_2d(st + StSmem::A, &tm_A, bar, 0, y);
        bulk_load(st + StSmem::DEC, ws.dec + sl * D, kDecBytes, bar);
    };
    if (tid == 0 && nch > 0) {
        prefetch_tmap(&tm_W);
        prefetch_tmap(&tm_U);
        prefetch_tmap(&tm_Q);
        prefetch_tmap(&tm_K);
        prefetch_tmap(&tm_A);
        issue(0);
    }
    // S <- S0 (or 0) in TMEM
#pragma unroll
    for (int cb = 0; cb < 8; ++cb) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = S0 ? S0[soff + cb * 16 + i] : 0.f;
        tmem_st16(tS + lane_base + cb * 16, v);
    }
    tmem_wait_st();

    uint32_t mma_phase = 0;
    for (int r = 0; r < nch; ++r) {
        uint8_t *st = sm + (r & 1) * StSmem::STAGE;
        const long tstart = t0 + (long)r * C;
        const int len = (int)min((long)C, t1 - tstart);
        if (tid == 0 && r + 1 < nch) {
            fence_proxy_async_smem();
            issue(r + 1);
        }
        {
            const bool ok = mbar_wait_bounded(&bars[r & 1], (r >> 1) & 1, kSpin, err);
            if (!__syncthreads_and(ok)) goto cleanup;
        }
        // S (fp32, TMEM) -> bf16 operand in smem; S <- S Diag(decay) in TMEM
        {
            const float *dec = reinterpret_cast<const float *>(st + StSmem::DEC);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[64];
#pragma unroll
                for (int cb = 0; cb < 4; ++cb)
                    tmem_ld16(tS + lane_base + half * 64 + cb * 16, v + cb * 16);
                tmem_wait_ld();
                uint8_t *rowp = sm + StSmem::S + half * 16384 + d * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4 *>(rowp + ((j ^ (d & 7)) << 4)) = pack8(v + j * 8);
#pragma unroll
                for (int i = 0; i < 64; ++i) v[i] *= dec[half * 64 + i];
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) tmem_st16(tS + lane_base + half * 64 + cb * 16, v + cb * 16);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk & 3) * 32;
                const uint64_t a =
                    sdesc_sw128(smem_u32(sm + StSmem::S + (kk >> 2) * 16384 + koff), 16, 1024);
                const uint64_t bw =
                    sdesc_sw128(smem_u32(st + StSmem::W + (kk >> 2) * 8192 + koff), 16, 1024);
                const uint64_t bq =
                    sdesc_sw128(smem_u32(st + StSmem::Q + (kk >> 2) * 8192 + koff), 16, 1024);
                mma_bf16_ss(tZ, a, bw, id, kk > 0);
                mma_bf16_ss(tO, a, bq, id, kk > 0);
            }
            mma_commit(&bars[2]);
        }
        {
            const bool ok = mbar_wait_bounded(&bars[2], mma_phase, kSpin, err);
            mma_phase ^= 1;
            if (!__syncthreads_and(ok)) goto cleanup;
        }
        tc_fence_after();
        // Z^T = U^T - S W<-^T  -> bf16 K-major operand in smem
        {
            float z[64];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) tmem_ld16(tZ + lane_base + cb * 16, z + cb * 16);
            tmem_wait_ld();
            const uint8_t *Ut = st + StSmem::U + (d >> 6) * 8192;
#pragma unroll
            for (int l = 0; l < 64; ++l) {
                const float u = __bfloat162float(
                    *reinterpret_cast<const __nv_bfloat16 *>(Ut + sw128_off(l, d & 63)));
                z[l] = u - z[l];
            }
            uint8_t *rowp = sm + StSmem::ZT + d * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(rowp + ((j ^ (d & 7)) << 4)) = pack8(z + j * 8);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idO = idesc_bf16(128, 64, 0, 0);
            const uint32_t idS = idesc_bf16(128, 128, 0, 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = sdesc_sw128(smem_u32(sm + StSmem::ZT + kk * 32), 16, 1024);
                const uint64_t ba = sdesc_sw128(smem_u32(st + StSmem::A + kk * 32), 16, 1024);
                const uint64_t bk = sdesc_sw128(smem_u32(st + StSmem::K + kk * 2048), 8192, 1024);
                mma_bf16_ss(tO, a, ba, idO, 1);
                mma_bf16_ss(tS, a, bk, idS, 1);
            }
            mma_commit(&bars[2]);
        }
        {
            const bool ok = mbar_wait_bounded(&bars[2], mma_phase, kSpin, err);
            mma_phase ^= 1;
            if (!__syncthreads_and(ok)) goto cleanup;
        }
        tc_fence_after();
        // O^T (TMEM) -> out[t, h, d]
        {
            __nv_bfloat16 *og = out + ((size_t)tstart * geo.H + h) * D + d;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float o[16];
                tmem_ld16(tO + lane_base + cb * 16, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int l = cb * 16 + i;
                    if (l < len) og[(size_t)l * geo.H * D] = __float2bfloat16_rn(o[i]);
                }
            }
        }
        __syncthreads();
    }
    if (S_final) {
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {
            float v[16];
            tmem_ld16(tS + lane_base + cb * 16, v);
            tmem_wait_ld();
            float4 *dst = reinterpret_cast<float4 *>(S_final + soff + cb * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
    }
cleanup:
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
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

WsLayout ws_layout(int B, int T, int H, int n_seq, int varlen) {
    WsLayout L;
    L.n_slots = varlen ? (T + C - 1) / C + n_seq : B * ((T + C - 1) / C);
    const size_t tiles = (size_t)L.n_slots * H;
    size_t o = 0;
    L.plan = o; o += up256(sizeof(int) * (size_t)(2 * (varlen ? n_seq : 0) + 1));
    L.dec = o;  o += up256(tiles * D * 4);
    L.W = o;    o += up256(tiles * C * D * 2);
    L.U = o;    o += up256(tiles * C * D * 2);
    L.Q = o;    o += up256(tiles * C * D * 2);
    L.K = o;    o += up256(tiles * C * D * 2);
    L.A = o;    o += up256(tiles * C * C * 2);
    L.total = o;
    return L;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    }
    return fn;
}

// 2-D bf16 tensor map: inner extent `inner` elements, `rows` rows, row pitch
// `pitch` bytes, box 64 x 64, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t pitch) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {pitch};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

size_t wy_smem_bytes(bool ch) {
    return 1024 + WySmem::end_tc(ch) + 4 * (64 * WySmem::NST + (ch ? 64 * D : 64) + 64) + 64;
}

}  // namespace

namespace gdr_host {

bool tc_applies(int dk, int dv, int chunk, gdr_dtype dtype) {
    return dtype == GDR_BF16 && dk == D && dv == D && chunk == C;
}

size_t tc_workspace_bytes(int B, int T, int H, int n_seq, int varlen, gdr_gate) {
    return ws_layout(B, T, H, n_seq, varlen).total;
}

cudaError_t fwd_tc_dispatch(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *S0, void *out, float *S_final, int B,
                            int T, int H, const int32_t *cu, int n_seq, gdr_gate gate,
                            void *workspace, size_t ws_bytes, unsigned int *err,
                            cudaStream_t st) {
    const int varlen = cu != nullptr;
    const WsLayout L = ws_layout(B, T, H, n_seq, varlen);
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

    const size_t tile_rows = (size_t)L.n_slots * H * C;
    if (tile_rows >= (size_t)1 << 31) return cudaErrorInvalidValue;  // 32-bit TMA row coordinates
    const uint64_t tok_rows = (uint64_t)B * T;
    CUtensorMap mq, mk, mv, mW, mU, mQ, mK, mA;
    const bool have_tokens = tok_rows > 0;
    if (have_tokens) {
        if (!make_map(&mq, q, (uint64_t)H * D, tok_rows, (uint64_t)H * D * 2) ||
            !make_map(&mk, k, (uint64_t)H * D, tok_rows, (uint64_t)H * D * 2) ||
            !make_map(&mv, v, (uint64_t)H * D, tok_rows, (uint64_t)H * D * 2) ||
            !make_map(&mW, ws.W, D, tile_rows, D * 2) || !make_map(&mU, ws.U, D, tile_rows, D * 2) ||
            !make_map(&mQ, ws.Q, D, tile_rows, D * 2) || !make_map(&mK, ws.K, D, tile_rows, D * 2) ||
            !make_map(&mA, ws.A, C, tile_rows, C * 2))
            return cudaErrorInvalidValue;
    } else {
        memset(&mW, 0, sizeof(mW));
        mU = mQ = mK = mA = mW;
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
        const size_t smem = wy_smem_bytes(ch);
        auto kern = ch ? wy_kernel<true> : wy_kernel<false>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        dim3 grid((unsigned)L.n_slots, (unsigned)H);
        ProfToken tk = prof_begin(GDR_K_TC_WY, st);
        kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, g, beta, cu, geo, ws, err);
        prof_end(tk, st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        const size_t smem = 1024 + StSmem::TOTAL;
        if ((e = cudaFuncSetAttribute(state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        ProfToken tk = prof_begin(GDR_K_TC_STATE, st);
        state_kernel<<<(unsigned)(geo.n_seq * H), kThreads, smem, st>>>(
            mW, mU, mQ, mK, mA, S0, (__nv_bfloat16 *)out, S_final, cu, geo, ws, err);
        prof_end(tk, st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdr_host
