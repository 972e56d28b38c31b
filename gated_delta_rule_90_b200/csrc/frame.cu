// Implicit frame-level update ("video-delta-rule", sections "A First Attempt at
// Frame-Level Updates" and "A Different Route").
//
// The tokens of a sequence are grouped into frames of n consecutive tokens
// (the last frame may be shorter).  Frame t has the erasure
// G_t = K_t^T Gamma K_t and the write C_t = V_t^T Gamma K_t (Gamma = diag of
// the tokens' writing strengths), and the state takes one implicit
// (backward-Euler) step
//     S_t (I + G_t) = S_{t-1} D_t + C_t,
// with the frame's decay D_t applied first (the forget gate sits at frame
// boundaries).  Every query of frame t reads S_t: o_i = S_t q_i.
//
// I + G_t is symmetric positive definite (the page factorises it by Cholesky
// and solves).  The step is affine in S_{t-1}:
//     S_t = (S_{t-1} D_t + C_t) W_t,   W_t = (I + G_t)^-1,
// and everything except the product chain over frames is independent per
// frame.  Four passes:
//   frame_gram    (frame, head, batch)    G_t, C_t                    fp32
//   frame_inverse (frame, head, batch)    W_t by the symmetric sweep
//                                         (Gauss-Jordan) of I + G_t
//   frame_chain   (batch*head, row block) S_t = (S_{t-1} D_t + C_t) W_t over
//                                         the frames (rows of S are independent)
//   frame_out     (token tile, head, batch) o_i = S_t q_i
// The inverse is fp32 on the CUDA cores.  For bf16 inputs with
// d_k = d_v = 128 the two dense contractions over tokens -- the Gram pass and
// the output pass -- run on the tensor cores (tcgen05, operands staged by TMA,
// fp32 accumulators in TMEM), and so does the chain, in a three-term bf16
// split that keeps its products at fp32 accuracy; otherwise all four passes
// are fp32 on the CUDA cores.
#include "common.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace gdr {
namespace frame {

using namespace sm100;
constexpr uint32_t kSpinF = 1u << 24;  // poll limit of every mbarrier wait

constexpr int kThreads = 256;
constexpr int kTokTile = 32;   // tokens per smem tile in the Gram and output passes
constexpr int kChainRows = 16; // state rows per CTA in the chain

struct Dims {
    int B, T, H, dk, dv, n, F;
};

__host__ __device__ inline size_t slot(const Dims &d, int b, int f, int h) {
    return ((size_t)b * d.F + f) * d.H + h;
}

// Checked build: (b, f, h) names a frame-head of the call, and the frames tile
// the T tokens (the last one may be shorter).  Every workspace slot a kernel
// touches is slot(d, b, f, h) of such a triple.
__device__ __forceinline__ bool frame_ok(const Dims &d, int b, int f, int h, unsigned int *err) {
    return chk_span(b, 1, d.B, err) && chk_span(f, 1, d.F, err) && chk_span(h, 1, d.H, err) &&
           chk_true(d.n >= 1 && (long long)(d.F - 1) * d.n < d.T && (long long)d.F * d.n >= d.T, err);
}

// G_t (d_k x d_k) then C_t (d_v x d_k): thread (ti, tj) owns an 8 x 8 block.
template <typename Tin>
__global__ void __launch_bounds__(kThreads)
frame_gram_kernel(const Tin *__restrict__ k, const Tin *__restrict__ v,
                  const float *__restrict__ gamma, float *__restrict__ Gw, float *__restrict__ Cw,
                  Dims d, unsigned int *err) {
    extern __shared__ float sm[];
    const int f = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    if (kChecked && !(frame_ok(d, b, f, h, err) && chk_true(d.dk <= 128 && d.dv <= 128, err))) return;
    const int kst = d.dk + 1, vst = d.dv + 1;
    float *Ks = sm, *Vs = Ks + kTokTile * kst, *gs = Vs + kTokTile * vst;
    const int tid = threadIdx.x, ti = tid >> 4, tj = tid & 15;
    const int t0 = f * d.n, t1 = min(d.T, t0 + d.n);
    const size_t sl = slot(d, b, f, h);
    for (int pass = 0; pass < 2; ++pass) {  // 0: G = K^T Gamma K, 1: C = V^T Gamma K
        const int rows = pass ? d.dv : d.dk;
        float acc[8][8];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;
        for (int tt = t0; tt < t1; tt += kTokTile) {
            const int cnt = min(kTokTile, t1 - tt);
            __syncthreads();
            for (int e = tid; e < kTokTile * d.dk; e += kThreads) {
                const int r = e / d.dk, c = e % d.dk;
                Ks[r * kst + c] = (r < cnt) ? ld_in(k, (((size_t)b * d.T + tt + r) * d.H + h) * d.dk + c) : 0.f;
            }
            if (pass)
                for (int e = tid; e < kTokTile * d.dv; e += kThreads) {
                    const int r = e / d.dv, c = e % d.dv;
                    Vs[r * vst + c] = (r < cnt) ? ld_in(v, (((size_t)b * d.T + tt + r) * d.H + h) * d.dv + c) : 0.f;
                }
            if (tid < kTokTile) gs[tid] = (tid < cnt) ? gamma[((size_t)b * d.T + tt + tid) * d.H + h] : 0.f;
            __syncthreads();
            if (ti * 8 < rows && tj * 8 < d.dk) {
                const float *Ls = pass ? Vs : Ks;
                const int lst = pass ? vst : kst;
                for (int r = 0; r < cnt; ++r) {
                    float x[8], y[8];
                    const float gr = gs[r];
#pragma unroll
                    for (int a = 0; a < 8; ++a) x[a] = gr * Ls[r * lst + ti * 8 + a];
#pragma unroll
                    for (int c = 0; c < 8; ++c) y[c] = Ks[r * kst + tj * 8 + c];
#pragma unroll
                    for (int a = 0; a < 8; ++a)
#pragma unroll
                        for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(x[a], y[c], acc[a][c]);
                }
            }
        }
        if (ti * 8 < rows && tj * 8 < d.dk) {
            float *dst = (pass ? Cw + sl * (size_t)d.dv * d.dk : Gw + sl * (size_t)d.dk * d.dk);
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int c = 0; c < 8; ++c) dst[(size_t)(ti * 8 + a) * d.dk + tj * 8 + c] = acc[a][c];
        }
    }
}

// W_t = (I + G_t)^-1 by the symmetric sweep (Gauss-Jordan) operator: sweeping
// pivot k maps a_kk -> -1/a_kk, a_ik -> a_ik / a_kk, a_kj -> a_kj / a_kk and
// a_ij -> a_ij - a_ik a_kj / a_kk; after every pivot the matrix is -(I + G_t)^-1.
// I + G_t is symmetric with eigenvalues >= 1, so every pivot (a Schur
// complement's diagonal) is >= 1 and no pivoting is needed.  G_t is
// symmetrised as (G + G^T) / 2 on load; with s = a_kk^-1/2 and c = s b (b =
// pivot row) the update a_ij -= c_i c_j is symmetric in i and j, so the matrix
// stays exactly symmetric and row k stands in for column k.  The pivot row
// passes through a double buffer in shared memory, written by the threads that
// hold it during the previous step: one barrier per pivot.  W_t overwrites
// G_t; with SPLIT it is written as two bf16 matrices instead, W_hi = bf16(W)
// and W_lo = bf16(W - W_hi), one after the other in the slot's first half (the
// operands of the tensor-core chain).
//
// The sweep runs on the upper triangle only: the update a_ij -= c_i c_j and
// the pivot's row and column give bit-identical values at (i, j) and (j, i),
// so a thread holds one 4 x 4 block (bi, bj), bi <= bj, of the upper triangle
// (a diagonal block in full), reads four pivot-row values for its rows and
// four for its columns, and mirrors the block on output (a layout of 4 x 8
// tiles over the whole matrix took 70 us against 64 us on the frame
// workload).  The next pivot row k + 1 is published by the blocks of block
// row (k + 1) / 4 (its columns from there on) and of block column (k + 1) / 4
// above the diagonal (its earlier columns, by symmetry).
constexpr int kSymThreads = 544;  // 17 warps >= 32 * 33 / 2 blocks (d_k = 128)

template <int DK, bool SPLIT>
__global__ void __launch_bounds__(kSymThreads, 2)
frame_inverse_sym_kernel(float *__restrict__ GW, Dims d, unsigned int *err) {
    constexpr int NB = DK / 4, NBLK = NB * (NB + 1) / 2;
    static_assert(NBLK <= kSymThreads, "one block per thread");
    __shared__ __align__(16) float buf[2][128];  // pivot rows
    const int f = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    if (kChecked && !(frame_ok(d, b, f, h, err) && chk_true(d.dk == DK, err))) return;
    const int tid = threadIdx.x;
    const bool act = tid < NBLK;
    int bi = 0, rem = tid;  // row-major enumeration of the upper-triangle blocks
    while (bi < NB && rem >= NB - bi) {
        rem -= NB - bi;
        ++bi;
    }
    const int bj = bi + rem, r0 = 4 * bi, c0 = 4 * bj;
    const size_t sl = slot(d, b, f, h);
    float *Gp = GW + sl * (size_t)DK * DK;
    float a[4][4];
    if (act) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 x = *reinterpret_cast<const float4 *>(Gp + (size_t)(r0 + i) * DK + c0);
            a[i][0] = x.x; a[i][1] = x.y; a[i][2] = x.z; a[i][3] = x.w;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // G^T: column c0 + u, rows r0..r0+3
            const float4 t = *reinterpret_cast<const float4 *>(Gp + (size_t)(c0 + u) * DK + r0);
            const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                a[i][u] = 0.5f * (a[i][u] + tv[i]) + (r0 + i == c0 + u ? 1.f : 0.f);
        }
        if (bi == 0)  // row 0 lies in block row 0
            *reinterpret_cast<float4 *>(&buf[0][c0]) = make_float4(a[0][0], a[0][1], a[0][2], a[0][3]);
    }
    __syncthreads();
    for (int k4 = 0; k4 < DK; k4 += 4) {
        const int kb = k4 >> 2;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int k = k4 + kk;
            const float *bk = buf[k & 1];
            const float dkk = bk[k];
            if (tid == 0 && !(dkk > 0.f)) atomicOr(err, kErrNumeric);
            const float sq = rsqrtf(dkk);
            if (act) {
                const float4 br = *reinterpret_cast<const float4 *>(bk + r0);
                const float4 bc = *reinterpret_cast<const float4 *>(bk + c0);
                const float cr[4] = {br.x * sq, br.y * sq, br.z * sq, br.w * sq};
                const float cc[4] = {bc.x * sq, bc.y * sq, bc.z * sq, bc.w * sq};
                const bool krow = kb == bi, kcol = kb == bj;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (krow && i == kk) {  // row k
#pragma unroll
                        for (int u = 0; u < 4; ++u) a[i][u] = (kcol && u == kk) ? -(sq * sq) : cc[u] * sq;
                    } else {
#pragma unroll
                        for (int u = 0; u < 4; ++u) a[i][u] = fmaf(-cr[i], cc[u], a[i][u]);
                        if (kcol) a[i][kk] = cr[i] * sq;  // column k
                    }
                }
                if (k + 1 < DK) {  // publish row k + 1
                    const int nb = (k + 1) >> 2, ni = (k + 1) & 3;
                    float *bn = buf[(k + 1) & 1];
                    if (bi == nb)
                        *reinterpret_cast<float4 *>(bn + c0) =
                            make_float4(a[ni][0], a[ni][1], a[ni][2], a[ni][3]);
                    else if (bj == nb)
                        *reinterpret_cast<float4 *>(bn + r0) =
                            make_float4(a[0][ni], a[1][ni], a[2][ni], a[3][ni]);
                }
            }
            __syncthreads();
        }
    }
    // the sweep leaves -W: the block and its mirror image
    if (act && !SPLIT) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4 *>(Gp + (size_t)(r0 + i) * DK + c0) =
                make_float4(-a[i][0], -a[i][1], -a[i][2], -a[i][3]);
        if (bi != bj) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                *reinterpret_cast<float4 *>(Gp + (size_t)(c0 + u) * DK + r0) =
                    make_float4(-a[0][u], -a[1][u], -a[2][u], -a[3][u]);
        }
    }
    if (act && SPLIT) {  // every read of G happened before the first barrier
        __nv_bfloat16 *wh = reinterpret_cast<__nv_bfloat16 *>(Gp), *wl = wh + DK * DK;
        auto split2 = [](float x, float y, uint32_t &hi, uint32_t &lo) {
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(-x, -y);
            const float2 hf = __bfloat1622float2(h2);
            const __nv_bfloat162 l2 = __floats2bfloat162_rn(-x - hf.x, -y - hf.y);
            hi = *reinterpret_cast<const uint32_t *>(&h2);
            lo = *reinterpret_cast<const uint32_t *>(&l2);
        };
        auto put = [&](int row, int col, float x0, float x1, float x2, float x3) {
            uint2 hv, lv;
            split2(x0, x1, hv.x, lv.x);
            split2(x2, x3, hv.y, lv.y);
            *reinterpret_cast<uint2 *>(wh + (size_t)row * DK + col) = hv;
            *reinterpret_cast<uint2 *>(wl + (size_t)row * DK + col) = lv;
        };
#pragma unroll
        for (int i = 0; i < 4; ++i) put(r0 + i, c0, a[i][0], a[i][1], a[i][2], a[i][3]);
        if (bi != bj) {
#pragma unroll
            for (int u = 0; u < 4; ++u) put(c0 + u, r0, a[0][u], a[1][u], a[2][u], a[3][u]);
        }
    }
}

static cudaError_t launch_inverse(float *GW, const Dims &d, bool split, unsigned int *err,
                                  cudaStream_t st) {
    const dim3 gf((unsigned)d.F, (unsigned)d.H, (unsigned)d.B);
    if (split) {
        if (d.dk != 128) return cudaErrorInvalidValue;
        frame_inverse_sym_kernel<128, true><<<gf, kSymThreads, 0, st>>>(GW, d, err);
        return cudaGetLastError();
    }
    switch (d.dk) {
#define GDR_INV(DK) \
    case DK: frame_inverse_sym_kernel<DK, false><<<gf, kSymThreads, 0, st>>>(GW, d, err); break
        GDR_INV(16); GDR_INV(32); GDR_INV(48); GDR_INV(64);
        GDR_INV(80); GDR_INV(96); GDR_INV(112); GDR_INV(128);
#undef GDR_INV
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// S_t = (S_{t-1} D_t + C_t) W_t for kChainRows rows of S in fp32 on the CUDA
// cores; every S_t is stored for the output pass, the last one also as S_final.  W_t arrives by bulk copy into one of two
// buffers, one frame ahead.  Thread (row pair rp = warp, column group cg =
// lane) owns rows 2 rp, 2 rp + 1 and columns 4 cg .. 4 cg + 3: each float4 read
// of a W_t row serves both rows (the chain is bound by shared-memory reads),
// and a warp's reads of S are broadcasts.
__global__ void __launch_bounds__(kThreads)
frame_chain_kernel(const float *__restrict__ Mw, const float *__restrict__ Cw,
                   const float *__restrict__ g, int per_channel,
                   const float *__restrict__ S0, float *__restrict__ Sw,
                   float *__restrict__ S_final, Dims d, unsigned int *err) {
    extern __shared__ __align__(16) float sm[];
    const int bh = blockIdx.x, b = bh / d.H, h = bh % d.H;
    const int r0 = blockIdx.y * kChainRows;
    const int nr = min(kChainRows, d.dv - r0);
    if (kChecked && !(frame_ok(d, b, 0, h, err) && chk_true(nr >= 1 && d.dk <= 128, err))) return;
    const int dk = d.dk, sst = dk + 4;
    // W_t double buffer (unpadded, as copied), then S rows [16][dk + 4]
    float *Mb = sm, *S = Mb + 2 * dk * dk;
    uint64_t *bar = reinterpret_cast<uint64_t *>(S + kChainRows * sst);  // [2]
    const int tid = threadIdx.x, rp = tid >> 5, cg = tid & 31, c4 = 4 * cg;
    const bool colok = c4 < dk;
    const bool mine0 = colok && 2 * rp < nr, mine1 = colok && 2 * rp + 1 < nr;
    const uint32_t mbytes = (uint32_t)(dk * dk * 4);
    const size_t soff = ((size_t)b * d.H + h) * (size_t)d.dv * dk;
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
    }
    for (int e = tid; e < kChainRows * dk; e += kThreads) {
        const int rr = e / dk, c = e % dk;
        S[rr * sst + c] = (S0 && rr < nr) ? S0[soff + (size_t)(r0 + rr) * dk + c] : 0.f;
    }
    __syncthreads();
    int issued = 0;
    if (tid == 0)
        for (; issued < 2 && issued < d.F; ++issued) {
            mbar_arrive_expect_tx(&bar[issued], mbytes);
            bulk_load(Mb + issued * dk * dk, Mw + slot(d, b, issued, h) * (size_t)dk * dk, mbytes,
                      &bar[issued]);
        }
    bool ok = true;
    float *Sr0 = S + (2 * rp) * sst, *Sr1 = Sr0 + sst;
    // C_t entries and log-decays of this thread's columns, loaded one frame
    // ahead so that their latency stays off the chain
    float4 cv0, cv1, gv;
    auto fetch = [&](int f) {
        const size_t sl = slot(d, b, f, h);
        const float *crow = Cw + sl * (size_t)d.dv * dk + (size_t)(r0 + 2 * rp) * dk + c4;
        cv0 = mine0 ? *reinterpret_cast<const float4 *>(crow) : make_float4(0.f, 0.f, 0.f, 0.f);
        cv1 = mine1 ? *reinterpret_cast<const float4 *>(crow + dk) : make_float4(0.f, 0.f, 0.f, 0.f);
        if (per_channel) {
            gv = *reinterpret_cast<const float4 *>(g + sl * dk + c4);
        } else {
            const float gs = g[sl];
            gv = make_float4(gs, gs, gs, gs);
        }
    };
    if (colok) fetch(0);
    for (int f = 0; f < d.F; ++f) {
        const size_t sl = slot(d, b, f, h);
        const float *Mf = Mb + (f & 1) * dk * dk;
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        if (colok) {  // S_{t-1} D_t + C_t, this thread's entries
            const float4 av = make_float4(expf(gv.x), expf(gv.y), expf(gv.z), expf(gv.w));
            float4 *p0 = reinterpret_cast<float4 *>(Sr0 + c4), *p1 = reinterpret_cast<float4 *>(Sr1 + c4);
            const float4 x0 = *p0, x1 = *p1;
            *p0 = make_float4(fmaf(x0.x, av.x, cv0.x), fmaf(x0.y, av.y, cv0.y), fmaf(x0.z, av.z, cv0.z),
                              fmaf(x0.w, av.w, cv0.w));
            *p1 = make_float4(fmaf(x1.x, av.x, cv1.x), fmaf(x1.y, av.y, cv1.y), fmaf(x1.z, av.z, cv1.z),
                              fmaf(x1.w, av.w, cv1.w));
            if (f + 1 < d.F) fetch(f + 1);
        }
        const bool okw = mbar_wait_bounded(&bar[f & 1], (f >> 1) & 1, kSpinF, err);
        if (!__syncthreads_and(okw)) { ok = false; break; }
        if (colok) {  // 4 rows of W_t per round, every load issued before the FMAs
            for (int m0 = 0; m0 < dk; m0 += 4) {
                const float4 s0 = *reinterpret_cast<const float4 *>(Sr0 + m0);
                const float4 s1 = *reinterpret_cast<const float4 *>(Sr1 + m0);
                const float sv0[4] = {s0.x, s0.y, s0.z, s0.w}, sv1[4] = {s1.x, s1.y, s1.z, s1.w};
                float4 w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) w[i] = *reinterpret_cast<const float4 *>(Mf + (m0 + i) * dk + c4);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float wv[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc0[j] = fmaf(sv0[i], wv[j], acc0[j]);
                        acc1[j] = fmaf(sv1[i], wv[j], acc1[j]);
                    }
                }
            }
        }
        __syncthreads();  // S and this W buffer are read
        if (tid == 0 && f + 2 < d.F) {
            mbar_arrive_expect_tx(&bar[f & 1], mbytes);
            bulk_load(Mb + (f & 1) * dk * dk, Mw + slot(d, b, f + 2, h) * (size_t)dk * dk, mbytes,
                      &bar[f & 1]);
            issued = f + 3;
        }
        if (colok) {
            *reinterpret_cast<float4 *>(Sr0 + c4) = make_float4(acc0[0], acc0[1], acc0[2], acc0[3]);
            *reinterpret_cast<float4 *>(Sr1 + c4) = make_float4(acc1[0], acc1[1], acc1[2], acc1[3]);
            const size_t o = sl * (size_t)d.dv * dk + (size_t)(r0 + 2 * rp) * dk + c4;
            if (mine0) *reinterpret_cast<float4 *>(Sw + o) = make_float4(acc0[0], acc0[1], acc0[2], acc0[3]);
            if (mine1) *reinterpret_cast<float4 *>(Sw + o + dk) = make_float4(acc1[0], acc1[1], acc1[2], acc1[3]);
        }
        __syncthreads();
    }
    if (ok && S_final && colok) {
        float *o = S_final + soff + (size_t)(r0 + 2 * rp) * dk + c4;
        if (mine0) *reinterpret_cast<float4 *>(o) = *reinterpret_cast<const float4 *>(Sr0 + c4);
        if (mine1) *reinterpret_cast<float4 *>(o + dk) = *reinterpret_cast<const float4 *>(Sr1 + c4);
    }
    if (tid == 0)  // copies still in flight (error path) land before exit
        for (int i = max(0, issued - 2); i < issued; ++i) mbar_wait_bounded(&bar[i & 1], (i >> 1) & 1, kSpinF, err);
}

// o_i = S_t q_i for a tile of kTokTile tokens inside one frame.
template <typename Tin>
__global__ void __launch_bounds__(kThreads)
frame_out_kernel(const Tin *__restrict__ q, const float *__restrict__ Sw, Tin *__restrict__ out,
                 Dims d, unsigned int *err) {
    extern __shared__ float sm[];
    const int tiles_per_frame = (d.n + kTokTile - 1) / kTokTile;
    const int f = blockIdx.x / tiles_per_frame, tile = blockIdx.x % tiles_per_frame;
    const int h = blockIdx.y, b = blockIdx.z;
    if (kChecked && !frame_ok(d, b, f, h, err)) return;
    const int tt = f * d.n + tile * kTokTile;
    const int cnt = min(kTokTile, min(d.T, (f + 1) * d.n) - tt);
    if (cnt <= 0) return;  // whole CTA, before any barrier
    const int dk = d.dk, ast = dk + 1;
    float *Ss = sm, *Qs = Ss + d.dv * ast;
    const int tid = threadIdx.x;
    const size_t sl = slot(d, b, f, h);
    for (int e = tid; e < d.dv * dk; e += kThreads) Ss[(e / dk) * ast + e % dk] = Sw[sl * (size_t)d.dv * dk + e];
    for (int e = tid; e < kTokTile * dk; e += kThreads) {
        const int r = e / dk, c = e % dk;
        Qs[r * ast + c] = (r < cnt) ? ld_in(q, (((size_t)b * d.T + tt + r) * d.H + h) * dk + c) : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < cnt * d.dv; e += kThreads) {
        const int r = e / d.dv, i = e % d.dv;
        float acc = 0.f;
        for (int m = 0; m < dk; ++m) acc = fmaf(Ss[i * ast + m], Qs[r * ast + m], acc);
        st_out(out, (((size_t)b * d.T + tt + r) * d.H + h) * d.dv + i, acc);
    }
}

// ---------------------------------------------------------------- tensor cores
constexpr int kTD = 128;                 // d_k = d_v on the tensor-core passes
constexpr int kGT = 64;                  // tokens per Gram tile (K = 64 per tile)
constexpr uint32_t kGStage = 3 * 16384;  // K, V, gamma . K (bf16, two 64-column atoms each)

// G_t = K^T (Gamma K) and C_t = V^T (Gamma K) on the tensor cores: M = N = 128
// (features), K = the frame's tokens, 64 per tile, two TMA stages.  K and V
// are MN-major A operands straight from their TMA tiles; Gamma K is a scaled
// copy (MN-major B).  Rows past the frame end get gamma = 0.
__global__ void __launch_bounds__(256)
frame_gram_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const float *__restrict__ gamma, float *__restrict__ Gw, float *__restrict__ Cw,
                     Dims d, unsigned int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + 2 * kGStage);  // [2]
    uint64_t *done = full + 2;                                         // [2]
    uint32_t *tslot = reinterpret_cast<uint32_t *>(done + 2);
    float *gs = reinterpret_cast<float *>(tslot + 4);                  // [2][64]
    const int f = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = f * d.n, t1 = min(d.T, t0 + d.n);
    const int ntiles = (t1 - t0 + kGT - 1) / kGT;
    const int x0 = h * kTD;
    const long yb = (long)b * d.T + t0;
    if (kChecked) {  // checked build: the frame-head, and its first and last token tiles
        const long long rows = (long long)d.B * d.T, xe = (long long)d.H * kTD;
        if (!(frame_ok(d, b, f, h, err) && chk_tma(x0 + 64, yb, 2, xe, rows, err) &&
              chk_tma(x0, yb + (long long)(ntiles - 1) * kGT, 2, xe, rows, err)))
            return;
    }
    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&done[0], 1);
        mbar_init(&done[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;  // G at [0,128), C at [128,256)
    auto issue = [&](int i) {
        uint8_t *st = sm + (i & 1) * kGStage;
        const int y = (int)(yb + (long)i * kGT);
        mbar_arrive_expect_tx(&full[i & 1], 4 * 8192);
        tma_load_2d(st, &tm_k, &full[i & 1], x0, y);
        tma_load_2d(st + 8192, &tm_k, &full[i & 1], x0 + 64, y);
        tma_load_2d(st + 16384, &tm_v, &full[i & 1], x0, y);
        tma_load_2d(st + 16384 + 8192, &tm_v, &full[i & 1], x0 + 64, y);
    };
    int issued = 0;  // tiles whose loads tid 0 issued
    if (tid == 0) {
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        for (; issued < 2 && issued < ntiles; ++issued) issue(issued);
    }
    bool ok = true;
    const uint32_t id = idesc_bf16(128, 128, 1, 1);
    for (int i = 0; i < ntiles; ++i) {
        const int s = i & 1;
        uint8_t *st = sm + s * kGStage;
        if (tid < kGT) {
            const int tok = t0 + i * kGT + tid;
            gs[s * kGT + tid] = (tok < t1) ? gamma[((size_t)b * d.T + tok) * d.H + h] : 0.f;
        }
        const bool okw = mbar_wait_bounded(&full[s], (i >> 1) & 1, kSpinF, err);
        if (!__syncthreads_and(okw)) { ok = false; break; }
        // gamma . K (element-wise, so the swizzled layout carries over)
        for (int e = tid; e < kGT * 16; e += 256) {
            const int r = e >> 4, c = e & 15;
            const uint32_t off = (c >> 3) * 8192 + r * 128 + (c & 7) * 16;
            float x[8];
            unpack8(*reinterpret_cast<const uint4 *>(st + off), x);
            const float gr = gs[s * kGT + r];
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] *= gr;
            *reinterpret_cast<uint4 *>(st + 32768 + off) = pack8(x);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dk_ = sdesc_sw128(smem_u32(st), 8192, 1024);
            const uint64_t dv_ = sdesc_sw128(smem_u32(st + 16384), 8192, 1024);
            const uint64_t dg_ = sdesc_sw128(smem_u32(st + 32768), 8192, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16_ss(tmem, sdesc_add(dk_, kk * 2048), sdesc_add(dg_, kk * 2048), id, (i | kk) > 0);
                mma_bf16_ss(tmem + 128, sdesc_add(dv_, kk * 2048), sdesc_add(dg_, kk * 2048), id, (i | kk) > 0);
            }
            mma_commit(&done[s]);
            if (i + 2 < ntiles) {  // this stage is free once its MMAs are done
                if (mbar_wait_bounded(&done[s], (i >> 1) & 1, kSpinF, err)) {
                    issue(i + 2);
                    issued = i + 3;
                }
            }
        }
    }
    // the last tile's MMAs cover all earlier ones
    if (ok && ntiles > 0) ok = mbar_wait_bounded(&done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, kSpinF, err);
    ok = __syncthreads_and(ok);  // the TMEM loads below are warp-wide: decide for all threads
    tc_fence_after();
    if (ok) {
        const int qd = warp & 3, hf = warp >> 2, row = qd * 32 + lane;
        const uint32_t lb = (uint32_t)(qd * 32) << 16;
        const size_t sl = slot(d, b, f, h);
        for (int m = 0; m < 2; ++m) {  // G, then C
            float *dst = (m ? Cw : Gw) + sl * (size_t)kTD * kTD + (size_t)row * kTD + hf * 64;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float x[16];
                if (ntiles > 0) {
                    tmem_ld16(tmem + m * 128 + lb + hf * 64 + cb * 16, x);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) x[j] = 0.f;
                }
                float4 *d4 = reinterpret_cast<float4 *>(dst + cb * 16);
#pragma unroll
                for (int j = 0; j < 4; ++j) d4[j] = make_float4(x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
            }
        }
    }
    // loads still in flight (error path) must land before the CTA exits
    if (tid == 0) {
        for (int i = max(0, issued - 2); i < issued; ++i) mbar_wait_bounded(&full[i & 1], (i >> 1) & 1, kSpinF, err);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// S_t = (S_{t-1} D_t + C_t) W_t on the tensor cores, for kCR rows of S per CTA.
// Rows of S are independent, and W_t is symmetric, so the step is computed
// transposed: S_t^T [128 x kCR] = W_t [128 x 128] * A_t^T with
// A_t = S_{t-1} D_t + C_t.  W_t is the K-major A operand, A_t^T the MN-major B
// operand (row m of it = key channel m over this CTA's rows of S), and the
// accumulator's TMEM lane j holds column j of S_t.  So a thread on TMEM lane j
// owns key channel j: its decay is one number, its C_t entries are column j of
// the CTA's row block, and its piece of the B operand is contiguous.
// kSplit threads share each channel (warps w, w + 4, ... reach the same TMEM
// lanes), each with kCR / kSplit of the rows.
//
// fp32 accuracy from bf16 products by the three-term split (Henry, Tang and
// Heinecke, "Leveraging the bfloat16 Artificial Intelligence Datatype For
// Higher-Precision Computations", 2019): x = x_hi + x_lo with x_hi = bf16(x),
// x_lo = bf16(x - x_hi), and
//     A W ~ A_hi W_hi + A_hi W_lo + A_lo W_hi
// (the dropped A_lo W_lo term is about 2^-16 of the product).  The inverse pass
// writes W_hi and W_lo; the chain splits A_t itself.  A_hi^T and A_lo^T sit
// side by side as one B operand of N = 2 kCR, so W_hi [A_hi^T A_lo^T] is one
// MMA per K step (accumulator columns [0, kCR) and [kCR, 2 kCR)), and
// W_lo A_hi^T adds into the first half: 16 MMAs per frame.
//
// Per frame: wait for the previous frame's MMAs, read S_{t-1} from TMEM (the
// sum of the two halves), form A_t and its two parts in shared memory, issue
// the MMAs, then -- while they run -- store S_{t-1} as the bf16 operand of the
// output pass (transposed, key channel major).  W_t (TMA, 64 KB) and the CTA's
// row block of C_t (one bulk copy, 32 KB) arrive together one frame ahead into
// one of two stages.
constexpr int kCR = 64;                      // rows of S per CTA
constexpr int kSplit = 4;                    // threads per key channel
constexpr int kChainThreads = 128 * kSplit;
constexpr int kHR = kCR / kSplit;            // rows per thread
constexpr int kWStages = 2;                  // stage ring depth
constexpr uint32_t kWBytes = 4 * 16384;      // W_hi, W_lo: two 64-column atoms each
constexpr uint32_t kCBytes = kCR * kTD * 4;  // C_t rows r0 .. r0 + kCR - 1, fp32
constexpr uint32_t kStage = kWBytes + kCBytes;
constexpr uint32_t kBBytes = 128 * kCR * 2;  // one part of A_t^T (MN-major, 128 B rows)
constexpr size_t kChainTcSmem = 1024 + kWStages * kStage + 2 * kBBytes + 64;
static_assert(kChainTcSmem <= 232448, "the chain's shared memory exceeds one CTA's limit");
static_assert(kCR == 64, "one 128-byte swizzle atom of A_t^T rows per part");
static_assert(kHR % 16 == 0, "whole 16-column TMEM loads per thread");

__global__ void __launch_bounds__(kChainThreads, 1)
frame_chain_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const float *__restrict__ Cw,
                      const float *__restrict__ g, int per_channel, const float *__restrict__ S0,
                      __nv_bfloat16 *__restrict__ Sb, float *__restrict__ S_final, Dims d,
                      unsigned int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *Bop = sm + kWStages * kStage;                                  // A_hi^T, then A_lo^T
    uint64_t *wfull = reinterpret_cast<uint64_t *>(Bop + 2 * kBBytes);      // [kWStages]
    uint64_t *mdone = wfull + kWStages;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(mdone + 1);
    const int bh = blockIdx.x, b = bh / d.H, h = bh % d.H;
    const int r0 = blockIdx.y * kCR;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int j = (warp & 3) * 32 + (tid & 31);  // key channel = TMEM lane
    const int hr = (warp >> 2) * kHR;            // this thread's rows: r0 + hr .. + kHR - 1
    const size_t soff = ((size_t)b * d.H + h) * (size_t)kTD * kTD;
    if (kChecked && !(frame_ok(d, b, 0, h, err) && chk_true(r0 + kCR <= kTD && d.dk == kTD && d.dv == kTD, err)))
        return;  // whole CTA, before any sync
    if (tid == 0) {
        for (int i = 0; i < kWStages; ++i) mbar_init(&wfull[i], 1);
        mbar_init(mdone, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 2 * kCR);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    const uint32_t tacc = tbase + ((uint32_t)((warp & 3) * 32) << 16) + hr;  // lanes, first column
    auto load_w = [&](int f) {  // W_hi rows at slot * 256, W_lo rows 128 further; C_t block
        const int st = f % kWStages;
        uint8_t *wb = sm + st * kStage;
        const size_t sl = slot(d, b, f, h);
        const int y = (int)(sl * 2 * kTD);
        mbar_arrive_expect_tx(&wfull[st], kStage);
        tma_load_2d(wb, &tm_w, &wfull[st], 0, y);
        tma_load_2d(wb + 16384, &tm_w, &wfull[st], 64, y);
        tma_load_2d(wb + 32768, &tm_w, &wfull[st], 0, y + kTD);
        tma_load_2d(wb + 49152, &tm_w, &wfull[st], 64, y + kTD);
        bulk_load(wb + kWBytes, Cw + (sl * kTD + r0) * (size_t)kTD, kCBytes, &wfull[st]);
    };
    int issued = 0, committed = 0;  // stage loads issued, frames whose MMAs were committed (tid 0)
    if (tid == 0) {
        prefetch_tmap(&tm_w);
        for (; issued < kWStages && issued < d.F; ++issued) load_w(issued);
    }
    float s[kHR];
#pragma unroll
    for (int r = 0; r < kHR; ++r) s[r] = S0 ? S0[soff + (size_t)(r0 + hr + r) * kTD + j] : 0.f;
    auto decay = [&](int f) {
        const size_t sl = slot(d, b, f, h);
        return per_channel ? g[sl * kTD + j] : g[sl];
    };
    float gj = decay(0);
    // this thread's piece of S_t^T (bf16, key channel major) for the output pass
    auto store_sb = [&](int f) {
        __nv_bfloat16 *o = Sb + (slot(d, b, f, h) * kTD + j) * kTD + r0 + hr;
#pragma unroll
        for (int q = 0; q < kHR / 8; ++q) reinterpret_cast<uint4 *>(o)[q] = pack8(s + 8 * q);
    };
    auto load_s = [&]() {  // S = columns [0, kCR) + columns [kCR, 2 kCR)
#pragma unroll
        for (int q = 0; q < kHR / 16; ++q) {
            float x[16];
            tmem_ld16(tacc + 16 * q, s + 16 * q);
            tmem_ld16(tacc + kCR + 16 * q, x);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) s[16 * q + u] += x[u];
        }
    };
    const uint32_t id2 = idesc_bf16(128, 2 * kCR, 0, 1), id1 = idesc_bf16(128, kCR, 0, 1);
    bool ok = true;
    for (int f = 0; f < d.F; ++f) {
        if (f > 0) {
            const bool okm = mbar_wait_bounded(mdone, (f - 1) & 1, kSpinF, err);
            if (!__syncthreads_and(okm)) { ok = false; break; }
            tc_fence_after();
            if (tid == 0 && f + kWStages - 1 < d.F) {  // frame f - 1's stage is free
                load_w(f + kWStages - 1);
                issued = f + kWStages;
            }
            load_s();
        }
        const int st = f % kWStages;
        const bool okw = mbar_wait_bounded(&wfull[st], (f / kWStages) & 1, kSpinF, err);
        if (!__syncthreads_and(okw)) { ok = false; break; }
        {  // A_t = S_{t-1} D_t + C_t, split; this thread's piece of row j of both parts
            const float dj = expf(gj);
            const float *cs = reinterpret_cast<const float *>(sm + st * kStage + kWBytes) + j;
#pragma unroll
            for (int q = 0; q < kHR / 8; ++q) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = 8 * q + 2 * u;
                    const float a0 = fmaf(s[r], dj, cs[(hr + r) * kTD]);
                    const float a1 = fmaf(s[r + 1], dj, cs[(hr + r + 1) * kTD]);
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(a0, a1);
                    const float2 hf = __bfloat1622float2(h2);
                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(a0 - hf.x, a1 - hf.y);
                    hi[u] = *reinterpret_cast<const uint32_t *>(&h2);
                    lo[u] = *reinterpret_cast<const uint32_t *>(&l2);
                }
                const int qg = (hr >> 3) + q;  // 16-byte chunk of the 128-byte row
                const uint32_t off = (uint32_t)(j * 128 + ((qg ^ (j & 7)) << 4));
                *reinterpret_cast<uint4 *>(Bop + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4 *>(Bop + kBBytes + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t wb = smem_u32(sm + st * kStage);
            const uint64_t dwh = sdesc_sw128(wb, 16, 1024), dwl = sdesc_sw128(wb + 32768, 16, 1024);
            const uint64_t db = sdesc_sw128(smem_u32(Bop), kBBytes, 1024);  // lbo: A_hi^T -> A_lo^T
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // W_hi [A_hi^T A_lo^T]
                mma_bf16_ss(tbase, sdesc_add(dwh, (kk >> 2) * 16384 + (kk & 3) * 32),
                            sdesc_add(db, kk * 2048), id2, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // + W_lo A_hi^T
                mma_bf16_ss(tbase, sdesc_add(dwl, (kk >> 2) * 16384 + (kk & 3) * 32),
                            sdesc_add(db, kk * 2048), id1, 1);
            mma_commit(mdone);
            committed = f + 1;
        }
        if (f > 0) store_sb(f - 1);  // s still holds S_{t-1}
        if (f + 1 < d.F) gj = decay(f + 1);
    }
    if (ok && d.F > 0) {
        ok = __syncthreads_and(mbar_wait_bounded(mdone, (d.F - 1) & 1, kSpinF, err));
        tc_fence_after();
        if (ok) {
            load_s();
            store_sb(d.F - 1);
            if (S_final)
#pragma unroll
                for (int r = 0; r < kHR; ++r) S_final[soff + (size_t)(r0 + hr + r) * kTD + j] = s[r];
        }
    }
    if (tid == 0) {  // work still in flight on an error path lands before TMEM and smem go
        if (committed > 0) mbar_wait_bounded(mdone, (committed - 1) & 1, kSpinF, err);
        for (int i = max(0, issued - kWStages); i < issued; ++i)
            mbar_wait_bounded(&wfull[i % kWStages], (i / kWStages) & 1, kSpinF, err);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 2 * kCR);
}

// o_i = S_t q_i for a tile of 128 tokens of one frame on the tensor cores:
// D[128 tokens x 128] = Q (K-major A) * S_t^T, the B operand being the chain's
// bf16 copy of S_t^T (key channel major, so MN-major: 64-column atoms 16 KB apart).
__global__ void __launch_bounds__(128)
frame_out_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_s,
                    __nv_bfloat16 *__restrict__ out, Dims d, unsigned int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + 65536);  // [2]: loads, MMAs
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bar + 2);
    const int tiles = (d.n + 127) / 128;
    const int f = blockIdx.x / tiles, tile = blockIdx.x % tiles;
    const int h = blockIdx.y, b = blockIdx.z;
    const int tt = f * d.n + tile * 128;
    const int cnt = min(128, min(d.T, (f + 1) * d.n) - tt);
    if (cnt <= 0) return;  // whole CTA, before any barrier
    if (kChecked && !(frame_ok(d, b, f, h, err) &&
                      chk_tma(h * kTD + 64, (long long)b * d.T + tt, 2, (long long)d.H * kTD,
                              (long long)d.B * d.T, err)))
        return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tslot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    // Q: two 64-feature atoms of [128 tokens][64]; S_t^T: two atoms of [128 rows (d_k)][64 (d_v)]
    if (tid == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_s);
        const int y = (int)((long)b * d.T + tt);
        const int ys = (int)(slot(d, b, f, h) * kTD);
        mbar_arrive_expect_tx(&bar[0], 65536);
        tma_load_2d(sm, &tm_q, &bar[0], h * kTD, y);
        tma_load_2d(sm + 8192, &tm_q, &bar[0], h * kTD, y + 64);
        tma_load_2d(sm + 16384, &tm_q, &bar[0], h * kTD + 64, y);
        tma_load_2d(sm + 16384 + 8192, &tm_q, &bar[0], h * kTD + 64, y + 64);
        tma_load_2d(sm + 32768, &tm_s, &bar[0], 0, ys);
        tma_load_2d(sm + 32768 + 16384, &tm_s, &bar[0], 64, ys);
    }
    bool ok = mbar_wait_bounded(&bar[0], 0, kSpinF, err);
    if (__syncthreads_and(ok) && tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, 128, 0, 1);
        const uint64_t da = sdesc_sw128(smem_u32(sm), 16, 1024);
        const uint64_t db = sdesc_sw128(smem_u32(sm + 32768), 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss(tmem, sdesc_add(da, (kk >> 2) * 16384 + (kk & 3) * 32),
                        sdesc_add(db, kk * 2048), id, kk > 0);
        mma_commit(&bar[1]);
    }
    ok = ok && mbar_wait_bounded(&bar[1], 0, kSpinF, err);
    ok = __syncthreads_and(ok);  // the TMEM loads below are warp-wide: decide for all threads
    tc_fence_after();
    if (ok) {  // thread = token row
        const int r = warp * 32 + lane;
        const uint32_t lb = (uint32_t)(warp * 32) << 16;
        __nv_bfloat16 *orow = out + (((size_t)b * d.T + tt + r) * d.H + h) * kTD;
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {
            float x[16];
            tmem_ld16(tmem + lb + cb * 16, x);
            tmem_wait_ld();
            if (r < cnt) {
                uint4 *o4 = reinterpret_cast<uint4 *>(orow + cb * 16);
                o4[0] = pack8(x);
                o4[1] = pack8(x + 8);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

}  // namespace frame
}  // namespace gdr

using namespace gdr;
using namespace gdr::frame;

namespace {

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

struct FrameLayout {
    // GM: G_t, overwritten by W_t (fp32; on the tensor-core path W_hi and W_lo in bf16)
    // CN: C_t (fp32)
    // Sw: fp32 S_t (on the tensor-core path bf16 S_t^T)
    size_t GM, CN, Sw, total;
};

FrameLayout frame_layout(int B, int T, int H, int dk, int dv, int n) {
    FrameLayout L;
    const size_t slots = (size_t)B * ((T + n - 1) / n) * H;
    size_t o = 0;
    L.GM = o; o += up256(slots * dk * dk * 4);
    L.CN = o; o += up256(slots * (size_t)dv * dk * 4);
    L.Sw = o; o += up256(slots * (size_t)dv * dk * 4);
    L.total = o;
    return L;
}

bool aligned16(const void *p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }

bool frame_shape_ok(int dk, int dv) {
    return dk >= 16 && dk <= 128 && dk % 16 == 0 && dv >= 8 && dv <= 128 && dv % 8 == 0;
}

bool frame_tc_applies(const Dims &d, bool bf16) { return bf16 && d.dk == kTD && d.dv == kTD; }

template <typename Tin>
cudaError_t frame_launch(const void *q, const void *k, const void *v, const float *g,
                         const float *gamma, const float *S0, void *out, float *S_final,
                         const Dims &d, int per_channel, uint8_t *ws, cudaStream_t st,
                         unsigned int *err) {
    const FrameLayout L = frame_layout(d.B, d.T, d.H, d.dk, d.dv, d.n);
    float *GM = (float *)(ws + L.GM), *CN = (float *)(ws + L.CN), *Sw = (float *)(ws + L.Sw);
    __nv_bfloat16 *Sb = (__nv_bfloat16 *)(ws + L.Sw);
    const bool tc = frame_tc_applies(d, sizeof(Tin) == 2);
    cudaError_t e;
    CUtensorMap mk, mv, mq, ms, mw;
    if (tc) {
        using namespace gdr_host::tmap;
        const uint64_t rows = (uint64_t)d.B * d.T, HD = (uint64_t)d.H * kTD;
        const uint64_t srows = (uint64_t)d.B * d.F * d.H * kTD;
        if (!make_map(&mk, kBF, k, HD, rows, HD * 2, 64, 64, kSW) ||
            !make_map(&mv, kBF, v, HD, rows, HD * 2, 64, 64, kSW) ||
            !make_map(&mq, kBF, q, HD, rows, HD * 2, 64, 64, kSW) ||
            !make_map(&ms, kBF, Sb, kTD, srows, kTD * 2, 64, 128, kSW) ||
            !make_map(&mw, kBF, GM, kTD, 2 * srows, kTD * 2, 64, 128, kSW))  // W_hi, W_lo per slot
            return cudaErrorInvalidValue;
    }
    const size_t sm_gram = sizeof(float) * (size_t)(kTokTile * (d.dk + 1) + kTokTile * (d.dv + 1) + kTokTile);
    const size_t sm_chain = sizeof(float) * (size_t)(2 * d.dk * d.dk + kChainRows * (d.dk + 4)) + 64;
    const size_t sm_out = sizeof(float) * (size_t)(d.dv + kTokTile) * (d.dk + 1);
    if ((e = cudaFuncSetAttribute(frame_gram_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_gram)) ||
        (e = cudaFuncSetAttribute(frame_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_chain)) ||
        (e = cudaFuncSetAttribute(frame_out_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_out)))
        return e;
    const dim3 gf((unsigned)d.F, (unsigned)d.H, (unsigned)d.B);
    const size_t sm_gram_tc = 1024 + 2 * kGStage + 1024, sm_out_tc = 1024 + 65536 + 64;
    if (tc &&
        ((e = cudaFuncSetAttribute(frame_gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_gram_tc)) ||
         (e = cudaFuncSetAttribute(frame_chain_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kChainTcSmem)) ||
         (e = cudaFuncSetAttribute(frame_out_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_out_tc))))
        return e;
    {
        gdr_host::ProfToken tk = gdr_host::prof_begin(GDR_K_FRAME_GRAM, st);
        if (tc)
            frame_gram_tc_kernel<<<gf, 256, sm_gram_tc, st>>>(mk, mv, gamma, GM, CN, d, err);
        else
            frame_gram_kernel<Tin><<<gf, kThreads, sm_gram, st>>>((const Tin *)k, (const Tin *)v, gamma, GM, CN, d, err);
        gdr_host::prof_end(tk, st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        gdr_host::ProfToken tk = gdr_host::prof_begin(GDR_K_FRAME_SOLVE, st);
        e = launch_inverse(GM, d, tc, err, st);
        gdr_host::prof_end(tk, st);
        if (e != cudaSuccess) return e;
    }
    {
        gdr_host::ProfToken tk = gdr_host::prof_begin(GDR_K_FRAME_CHAIN, st);
        if (tc) {
            const dim3 gc((unsigned)(d.B * d.H), (unsigned)(kTD / kCR));
            frame_chain_tc_kernel<<<gc, kChainThreads, kChainTcSmem, st>>>(mw, CN, g, per_channel, S0,
                                                                           Sb, S_final, d, err);
        } else {
            const dim3 gc((unsigned)(d.B * d.H), (unsigned)((d.dv + kChainRows - 1) / kChainRows));
            frame_chain_kernel<<<gc, kThreads, sm_chain, st>>>(GM, CN, g, per_channel, S0, Sw,
                                                               S_final, d, err);
        }
        gdr_host::prof_end(tk, st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        gdr_host::ProfToken tk = gdr_host::prof_begin(GDR_K_FRAME_OUT, st);
        if (tc) {
            const dim3 go((unsigned)(d.F * ((d.n + 127) / 128)), (unsigned)d.H, (unsigned)d.B);
            frame_out_tc_kernel<<<go, 128, sm_out_tc, st>>>(mq, ms, (__nv_bfloat16 *)out, d, err);
        } else {
            const int tiles = (d.n + kTokTile - 1) / kTokTile;
            const dim3 go((unsigned)(d.F * tiles), (unsigned)d.H, (unsigned)d.B);
            frame_out_kernel<Tin><<<go, kThreads, sm_out, st>>>((const Tin *)q, Sw, (Tin *)out, d, err);
        }
        gdr_host::prof_end(tk, st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t gdr_fwd_frame_workspace_size(int B, int T, int H, int d_k, int d_v, int n) {
    if (B < 1 || T < 1 || H < 1 || n < 1 || !frame_shape_ok(d_k, d_v)) return 0;
    return frame_layout(B, T, H, d_k, d_v, n).total;
}

gdr_status gdr_fwd_frame(const void *q, const void *k, const void *v, const float *g,
                         const float *gamma, const float *S0, void *out, float *S_final, int B,
                         int T, int H, int d_k, int d_v, int n, gdr_dtype dtype, gdr_gate gate,
                         void *workspace, size_t workspace_bytes, void *stream) {
    if (B < 1 || T < 0 || H < 1 || d_k < 1 || d_v < 1 || n < 1) return GDR_ERR_INVALID;
    if (!(dtype == GDR_F32 || dtype == GDR_BF16) ||
        !(gate == GDR_GATE_SCALAR || gate == GDR_GATE_PER_KEY_CHANNEL))
        return GDR_ERR_INVALID;
    if (!frame_shape_ok(d_k, d_v)) return GDR_ERR_UNSUPPORTED;
    if ((double)B * T * H * (d_k > d_v ? d_k : d_v) > 9.0e15 || (double)B * T > 2.0e9 ||
        (double)B * H * ((T + n - 1) / n) > 2.0e9)
        return GDR_ERR_INVALID;
    if (B > 65535 || H > 65535) return GDR_ERR_UNSUPPORTED;  // grid y / z extents
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(gamma) ||
        !aligned16(S0) || !aligned16(out) || !aligned16(S_final) || !aligned16(workspace))
        return GDR_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    if (T == 0) {  // no frames: the state passes through
        if (S_final && S0 != S_final) {
            const size_t bytes = sizeof(float) * (size_t)B * H * d_v * d_k;
            cudaError_t e = S0 ? cudaMemcpyAsync(S_final, S0, bytes, cudaMemcpyDeviceToDevice, st)
                               : cudaMemsetAsync(S_final, 0, bytes, st);
            return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
        }
        return GDR_OK;
    }
    if (!q || !k || !v || !g || !gamma || !out) return GDR_ERR_INVALID;
    const FrameLayout L = frame_layout(B, T, H, d_k, d_v, n);
    if (!workspace || workspace_bytes < L.total) return GDR_ERR_INVALID;
    Dims d{B, T, H, d_k, d_v, n, (T + n - 1) / n};
    unsigned int *err = gdr_host::device_error_word();
    if (!err) return GDR_ERR_CUDA;
    const int ch = gate == GDR_GATE_PER_KEY_CHANNEL;
    cudaError_t e = dtype == GDR_BF16
                        ? frame_launch<__nv_bfloat16>(q, k, v, g, gamma, S0, out, S_final, d, ch,
                                                      (uint8_t *)workspace, st, err)
                        : frame_launch<float>(q, k, v, g, gamma, S0, out, S_final, d, ch,
                                              (uint8_t *)workspace, st, err);
    return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

}  // extern "C"
