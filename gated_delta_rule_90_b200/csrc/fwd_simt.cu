// SIMT (fp32 CUDA-core) chunkwise prefill of the gated delta rule.
//
// The path for fp32 inputs (where bf16 tensor-core operands would not meet an
// fp32 tolerance) and for shapes outside the tensor-core path; it is also the
// GPU-side cross-check of that path.  One CTA owns one (sequence, head, slice of
// 32 state rows) and walks the sequence's chunks in order.  Per chunk r it takes
// the steps of "Linear Attention, Visualized", "Gated DeltaNet (GDN) / Complete
// per-chunk algorithm" and "Kimi Delta Attention (KDA) / Complete per-chunk
// algorithm", transposed to the column convention (S is d_v x d_k; only the
// CTA's rows of S are held):
//   G_l       = sum_{s<=l} g_s                       (cumulative log-decay)
//   L[l,m]    = sum_c k_lc k_mc exp(G_lc - G_mc)      (m < l)
//   A[l,m]    = sum_c q_lc k_mc exp(G_lc - G_mc)      (m <= l)
//   (I + diag(beta) L) T = diag(beta)                 (column-wise forward substitution)
//   Z         = T (V - K<- S^T)          (= U - W<- S^T with U = T V, W<- = T K<-)
//   O         = Q<- S^T + A Z
//   S         <- S Diag(exp(G_C)) + Z^T K->
// with K<- = exp(G) . K, Q<- = exp(G) . Q, K-> = exp(G_C - G) . K.  Decay ratios
// are always formed as exp of a difference of cumulative sums, never as a ratio
// of products.  A chunk that runs past the end of its sequence treats the
// missing tokens as k = q = v = 0, beta = 0, g = 0, which leaves every valid
// row unchanged (the pages assume the chunk size divides the length).
//
// With DEC (Gated DeltaNet-2, "Gated DeltaNet-2, and the gate that was doing
// two jobs", section "What decoupling actually means here") beta splits into an
// erase gate b (per key channel) and a write gate w (per value channel):
// e = b . k, z = w . v.  The same chunk algorithm then reads
//   L[l,m]  = sum_c e_lc k_mc exp(G_lc - G_mc)   (m < l),  (I + L) T = I,
//   Z       = T (w . V - E<- S^T),   E<- = exp(G) . E,
// and O, S as above: the erase vector replaces beta k on the reading side, the
// key stays the writing direction.
#include "common.cuh"

namespace gdr {

constexpr int kSimtThreads = 256;
constexpr int kSimtRows = 32;  // state rows (d_v) per CTA

struct SimtSmem {
    // offsets in floats
    int Kc, Qc, Gc, Kx, bt, kd, Nm, Am, Tm, Pm, Zm, Ss, total;
    int kst;  // padded row stride of the [C][d_k] buffers
};

__host__ __device__ inline SimtSmem simt_layout(int C, int dk, bool channel, bool dec) {
    SimtSmem L;
    L.kst = dk + 1;
    int o = 0;
    L.Kc = o; o += C * L.kst;
    L.Qc = o; o += C * L.kst;
    L.Gc = o; o += channel ? C * L.kst : C;
    L.Kx = o; o += (channel || dec) ? C * L.kst : 0;  // K<- / E<-, then K->
    L.bt = o; o += C;
    L.kd = o; o += C;  // scalar gate: e^(G_C - G_l) per row
    L.Nm = o; o += C * C;
    L.Am = o; o += C * C;
    L.Tm = o; o += C * C;
    L.Pm = o; o += C * kSimtRows;
    L.Zm = o; o += C * kSimtRows;
    L.Ss = o; o += kSimtRows * L.kst;
    L.total = o;
    return L;
}

template <typename Tin, bool CH, bool DEC>
__global__ void __launch_bounds__(kSimtThreads)
fwd_simt_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                const float *__restrict__ g, const float *__restrict__ beta,
                const float *__restrict__ eg, const float *__restrict__ wg,
                const float *__restrict__ S0, Tin *__restrict__ out, float *__restrict__ S_final,
                int T, int H, int dk, int dv, int C, const int32_t *__restrict__ cu, int T_total,
                int n_seq, unsigned int *err) {
    extern __shared__ float sm[];
    const SimtSmem L = simt_layout(C, dk, CH, DEC);
    float *Kc = sm + L.Kc, *Qc = sm + L.Qc, *Gc = sm + L.Gc, *Kx = sm + L.Kx, *bt = sm + L.bt;
    float *kd = sm + L.kd;
    float *Nm = sm + L.Nm, *Am = sm + L.Am, *Tm = sm + L.Tm, *Pm = sm + L.Pm, *Zm = sm + L.Zm;
    float *Ss = sm + L.Ss;
    const int kst = L.kst;
    const int tid = threadIdx.x;
    const int s = blockIdx.x / H, h = blockIdx.x % H;
    const int r0 = blockIdx.y * kSimtRows;
    const int nr = min(kSimtRows, dv - r0);
    long t0, t1;
    seq_bounds(cu, s, T, T_total, t0, t1);
    if (kChecked) {  // checked build: this CTA's tokens, state rows and state slot
        const long long rows = cu ? (long long)T_total : (long long)n_seq * T;
        if (!(chk_span(s, 1, n_seq, err) && chk_span(t0, t1 - t0, rows, err) &&
              chk_true(nr >= 1 && r0 + nr <= dv, err)))
            return;
    }

    // state slice: rows r0 .. r0+nr of S (d_v x d_k)
    const size_t soff = ((size_t)s * H + h) * (size_t)dv * dk;
    for (int e = tid; e < kSimtRows * dk; e += kSimtThreads) {
        const int r = e / dk, c = e % dk;
        Ss[r * kst + c] = (S0 && r < nr) ? S0[soff + (size_t)(r0 + r) * dk + c] : 0.f;
    }

    for (long c0 = t0; c0 < t1; c0 += C) {
        const int len = (int)min((long)C, t1 - c0);
        __syncthreads();
        // ---- load the chunk (missing tokens are zero) ----
        for (int e = tid; e < C * dk; e += kSimtThreads) {
            const int l = e / dk, c = e % dk;
            float kv = 0.f, qv = 0.f;
            if (l < len) {
                const size_t off = ((size_t)(c0 + l) * H + h) * dk + c;
                kv = ld_in(k, off);
                qv = ld_in(q, off);
            }
            Kc[l * kst + c] = kv;
            Qc[l * kst + c] = qv;
            if (CH) Gc[l * kst + c] = (l < len) ? g[((size_t)(c0 + l) * H + h) * dk + c] : 0.f;
            if (DEC) Kx[l * kst + c] = (l < len) ? kv * eg[((size_t)(c0 + l) * H + h) * dk + c] : 0.f;
        }
        for (int l = tid; l < C; l += kSimtThreads) {
            const size_t off = (size_t)(c0 + l) * H + h;
            bt[l] = (l < len) ? (DEC ? 1.f : beta[off]) : 0.f;
            if (!CH) Gc[l] = (l < len) ? g[off] : 0.f;
        }
        __syncthreads();
        // ---- cumulative log-decay G (in place) ----
        if (CH) {
            for (int c = tid; c < dk; c += kSimtThreads) {
                float acc = 0.f;
                for (int l = 0; l < C; ++l) {
                    acc += Gc[l * kst + c];
                    Gc[l * kst + c] = acc;
                }
            }
        } else if (tid == 0) {
            float acc = 0.f;
            for (int l = 0; l < C; ++l) {
                acc += Gc[l];
                Gc[l] = acc;
            }
        }
        __syncthreads();
        // ---- L (scaled by beta into N = diag(beta) L) and A ----
        for (int p = tid; p < C * C; p += kSimtThreads) {
            const int l = p / C, m = p % C;
            float lv = 0.f, av = 0.f;
            if (m <= l) {
                // reading side: the key (beta applied below) or the erase vector
                const float *kl = (DEC ? Kx : Kc) + l * kst, *km = Kc + m * kst, *ql = Qc + l * kst;
                if (CH) {
                    const float *gl = Gc + l * kst, *gm = Gc + m * kst;
                    for (int c = 0; c < dk; ++c) {
                        const float w = km[c] * expf(gl[c] - gm[c]);
                        lv = fmaf(kl[c], w, lv);
                        av = fmaf(ql[c], w, av);
                    }
                } else {
                    for (int c = 0; c < dk; ++c) {
                        lv = fmaf(kl[c], km[c], lv);
                        av = fmaf(ql[c], km[c], av);
                    }
                    const float w = expf(Gc[l] - Gc[m]);
                    lv *= w;
                    av *= w;
                }
            }
            Nm[p] = (m < l) ? bt[l] * lv : 0.f;
            Am[p] = av;
        }
        __syncthreads();
        // ---- T: (I + N) T = diag(beta), thread j solves column j ----
        for (int j = tid; j < C; j += kSimtThreads) {
            for (int i = 0; i < C; ++i) {
                float acc = (i == j) ? bt[j] : 0.f;
                for (int m = 0; m < i; ++m) acc = fmaf(-Nm[i * C + m], Tm[m * C + j], acc);
                Tm[i * C + j] = (i < j) ? 0.f : acc;
            }
        }
        // decayed copies: Q<- in place; K<- into Kx (per channel), or E<- in
        // place in Kx (erase vectors) -- A and L are done
        for (int e = tid; e < C * dk; e += kSimtThreads) {
            const int l = e / dk, c = e % dk;
            const float w = expf(CH ? Gc[l * kst + c] : Gc[l]);
            Qc[l * kst + c] *= w;
            if (DEC) Kx[l * kst + c] *= w;
            else if (CH) Kx[l * kst + c] = Kc[l * kst + c] * w;
        }
        __syncthreads();
        // ---- P = V - K<- S^T  (C x nr) ----
        for (int e = tid; e < C * kSimtRows; e += kSimtThreads) {
            const int l = e / kSimtRows, r = e % kSimtRows;
            float acc = 0.f;
            if (r < nr && l < len) {
                const float *kl = (CH || DEC) ? Kx + l * kst : Kc + l * kst;
                const float *sr = Ss + r * kst;
                for (int c = 0; c < dk; ++c) acc = fmaf(kl[c], sr[c], acc);
                if (!CH && !DEC) acc *= expf(Gc[l]);
                const size_t vo = ((size_t)(c0 + l) * H + h) * dv + r0 + r;
                acc = (DEC ? ld_in(v, vo) * wg[vo] : ld_in(v, vo)) - acc;
            }
            Pm[e] = acc;
        }
        __syncthreads();
        // ---- Z = T P ----
        for (int e = tid; e < C * kSimtRows; e += kSimtThreads) {
            const int l = e / kSimtRows, r = e % kSimtRows;
            float acc = 0.f;
            for (int m = 0; m <= l; ++m) acc = fmaf(Tm[l * C + m], Pm[m * kSimtRows + r], acc);
            Zm[e] = acc;
        }
        __syncthreads();
        // ---- O = Q<- S^T + A Z ----
        for (int e = tid; e < C * kSimtRows; e += kSimtThreads) {
            const int l = e / kSimtRows, r = e % kSimtRows;
            if (r < nr && l < len) {
                float acc = 0.f;
                const float *ql = Qc + l * kst, *sr = Ss + r * kst;
                for (int c = 0; c < dk; ++c) acc = fmaf(ql[c], sr[c], acc);
                for (int m = 0; m <= l; ++m) acc = fmaf(Am[l * C + m], Zm[m * kSimtRows + r], acc);
                st_out(out, ((size_t)(c0 + l) * H + h) * dv + r0 + r, acc);
            }
        }
        // K-> = exp(G_C - G) . K into Kx (Kx's K<- is no longer read after P)
        const int last = C - 1;
        if (CH) {
            for (int e = tid; e < C * dk; e += kSimtThreads) {
                const int l = e / dk, c = e % dk;
                Kx[l * kst + c] = Kc[l * kst + c] * expf(Gc[last * kst + c] - Gc[l * kst + c]);
            }
        } else {  // the scalar gate's write factors, once per row
            for (int l = tid; l < C; l += kSimtThreads) kd[l] = expf(Gc[last] - Gc[l]);
        }
        __syncthreads();
        // ---- S <- S Diag(exp(G_C)) + Z^T K-> ----
        for (int e = tid; e < kSimtRows * dk; e += kSimtThreads) {
            const int r = e / dk, c = e % dk;
            float acc;
            if (CH) {
                acc = Ss[r * kst + c] * expf(Gc[last * kst + c]);
                for (int l = 0; l < C; ++l) acc = fmaf(Zm[l * kSimtRows + r], Kx[l * kst + c], acc);
            } else {
                acc = Ss[r * kst + c] * expf(Gc[last]);
                for (int l = 0; l < C; ++l) acc = fmaf(Zm[l * kSimtRows + r] * kd[l], Kc[l * kst + c], acc);
            }
            Ss[r * kst + c] = acc;
        }
    }
    __syncthreads();
    if (S_final) {
        for (int e = tid; e < nr * dk; e += kSimtThreads) {
            const int r = e / dk, c = e % dk;
            S_final[soff + (size_t)(r0 + r) * dk + c] = Ss[r * kst + c];
        }
    }
}

// ------------------------------------------------------------------ wide chunks
// The same chunk algorithm for chunks whose resident tiles do not fit in
// shared memory (C = 128 with d_k = 128 would need 380 to 510 KB above).
// Only the C x C matrices, the CTA's state rows and the P/Z tiles stay
// resident; the chunk's key-side inputs (k, q, g and the erase vectors) pass
// through shared memory in blocks of kWideKB key channels, twice per chunk:
//   pass 1, per block: L and A accumulate their partial channel sums (the
//           decay ratio exp(G_lc - G_mc) formed per channel as above), then the
//           block is decayed in place and K<- S^T, Q<- S^T accumulate in
//           registers;
//   solve:  (I + N) T = diag(beta) column by column, T stored transposed in
//           the strict upper triangle of N's buffer (T's diagonal is beta);
//   Z = T P, O = Q<- S^T + A Z;
//   pass 2, per block: K-> formed in place, S's columns of the block updated.
// Every product is the one the resident kernel forms; only the order of the
// channel sums differs.
constexpr int kWideKB = 16;    // key channels per block
constexpr int kWideMaxC = 128;
constexpr int kWideRegs = kWideMaxC * kSimtRows / kSimtThreads;  // P / Q<-S^T entries per thread
constexpr int kWideSegs = kSimtThreads / kWideKB;                // scan segments per channel

struct WideSmem {
    int NT, Am, Kb, Qb, Gb, Eb, Pm, Zm, Ss, bt, Gs, seg, total;
    int bst, sst;  // row strides of the channel blocks and of the state rows
};

__host__ __device__ inline WideSmem wide_layout(int C, int dk, bool channel, bool dec) {
    WideSmem L;
    L.bst = kWideKB + 1;
    L.sst = dk + 1;
    int o = 0;
    L.NT = o; o += C * C;
    L.Am = o; o += C * C;
    L.Kb = o; o += C * L.bst;
    L.Qb = o; o += C * L.bst;
    L.Gb = o; o += channel ? C * L.bst : 0;
    L.Eb = o; o += dec ? C * L.bst : 0;
    L.Pm = o; o += C * kSimtRows;
    L.Zm = o; o += C * kSimtRows;
    L.Ss = o; o += kSimtRows * L.sst;
    L.bt = o; o += C;
    L.Gs = o; o += C;
    L.seg = o; o += kWideSegs * kWideKB;
    L.total = o;
    return L;
}

// Row l and column m (m <= l) of the p-th entry of a row-major lower triangle.
__device__ __forceinline__ void tri_index(int p, int &l, int &m) {
    int r = (int)((sqrtf(8.f * (float)p + 1.f) - 1.f) * 0.5f);
    while ((r + 1) * (r + 2) / 2 <= p) ++r;
    while (r * (r + 1) / 2 > p) --r;
    l = r;
    m = p - r * (r + 1) / 2;
}

template <typename Tin, bool CH, bool DEC>
__global__ void __launch_bounds__(kSimtThreads)
fwd_simt_wide_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                     const float *__restrict__ g, const float *__restrict__ beta,
                     const float *__restrict__ eg, const float *__restrict__ wg,
                     const float *__restrict__ S0, Tin *__restrict__ out, float *__restrict__ S_final,
                     int T, int H, int dk, int dv, int C, const int32_t *__restrict__ cu,
                     int T_total, int n_seq, unsigned int *err) {
    extern __shared__ float sm[];
    const WideSmem L = wide_layout(C, dk, CH, DEC);
    float *NT = sm + L.NT, *Am = sm + L.Am, *Kb = sm + L.Kb, *Qb = sm + L.Qb, *Gb = sm + L.Gb;
    float *Eb = sm + L.Eb, *Pm = sm + L.Pm, *Zm = sm + L.Zm, *Ss = sm + L.Ss, *bt = sm + L.bt;
    float *Gs = sm + L.Gs, *seg = sm + L.seg;
    const int bst = L.bst, sst = L.sst;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int s = blockIdx.x / H, h = blockIdx.x % H;
    const int r0 = blockIdx.y * kSimtRows;
    const int nr = min(kSimtRows, dv - r0);
    const int npairs = C * (C + 1) / 2;
    const int seglen = (C + kWideSegs - 1) / kWideSegs;
    long t0, t1;
    seq_bounds(cu, s, T, T_total, t0, t1);
    if (kChecked) {  // checked build: this CTA's tokens, state rows and state slot
        const long long rows = cu ? (long long)T_total : (long long)n_seq * T;
        if (!(chk_span(s, 1, n_seq, err) && chk_span(t0, t1 - t0, rows, err) &&
              chk_true(nr >= 1 && r0 + nr <= dv, err)))
            return;
    }

    const size_t soff = ((size_t)s * H + h) * (size_t)dv * dk;
    for (int e = tid; e < kSimtRows * dk; e += kSimtThreads) {
        const int r = e / dk, c = e % dk;
        Ss[r * sst + c] = (S0 && r < nr) ? S0[soff + (size_t)(r0 + r) * dk + c] : 0.f;
    }

    // Load channels [cb, cb + kWideKB) of the chunk's keys (and queries, gate,
    // erase vectors); with CH the gate block becomes its cumulative sum over
    // the chunk.  Ends with the block visible to the whole CTA.
    auto load_block = [&](long c0, int len, int cb, bool with_q) {
        for (int i = tid; i < C * kWideKB; i += kSimtThreads) {
            const int l = i / kWideKB, c = i % kWideKB;
            float kv = 0.f, qv = 0.f, gv = 0.f, ev = 0.f;
            if (l < len) {
                const size_t off = ((size_t)(c0 + l) * H + h) * dk + cb + c;
                kv = ld_in(k, off);
                if (with_q) qv = ld_in(q, off);
                if (CH) gv = g[off];
                if (DEC) ev = kv * eg[off];
            }
            Kb[l * bst + c] = kv;
            if (with_q) Qb[l * bst + c] = qv;
            if (CH) Gb[l * bst + c] = gv;
            if (DEC) Eb[l * bst + c] = ev;
        }
        __syncthreads();
        if (CH) {  // segmented scan: channel tid % KB, rows of segment tid / KB
            const int c = tid % kWideKB, sg = tid / kWideKB;
            const int la = sg * seglen, lb = min(C, la + seglen);
            float acc = 0.f;
            for (int l = la; l < lb; ++l) {
                acc += Gb[l * bst + c];
                Gb[l * bst + c] = acc;
            }
            seg[sg * kWideKB + c] = acc;
            __syncthreads();
            float pre = 0.f;
            for (int j = 0; j < sg; ++j) pre += seg[j * kWideKB + c];
            for (int l = la; l < lb; ++l) Gb[l * bst + c] += pre;
            __syncthreads();
        }
    };

    for (long c0 = t0; c0 < t1; c0 += C) {
        const int len = (int)min((long)C, t1 - c0);
        __syncthreads();  // the previous chunk is done with every buffer
        for (int l = tid; l < C; l += kSimtThreads) {
            const size_t off = (size_t)(c0 + l) * H + h;
            bt[l] = (l < len) ? (DEC ? 1.f : beta[off]) : 0.f;
            if (!CH) Gs[l] = (l < len) ? g[off] : 0.f;
        }
        __syncthreads();
        if (!CH && tid == 0) {
            float acc = 0.f;
            for (int l = 0; l < C; ++l) {
                acc += Gs[l];
                Gs[l] = acc;
            }
        }
        // ---- pass 1: L, A (shared memory), K<- S^T and Q<- S^T (registers) ----
        float pacc[kWideRegs], qacc[kWideRegs];
#pragma unroll
        for (int i = 0; i < kWideRegs; ++i) pacc[i] = qacc[i] = 0.f;
        const float *Rb = DEC ? Eb : Kb;  // reading direction
        for (int cb = 0; cb < dk; cb += kWideKB) {
            load_block(c0, len, cb, true);
            for (int p = tid; p < npairs; p += kSimtThreads) {
                int l, m;
                tri_index(p, l, m);
                float lv = 0.f, av = 0.f;
#pragma unroll 4
                for (int c = 0; c < kWideKB; ++c) {
                    float w = Kb[m * bst + c];
                    if (CH) w *= expf(Gb[l * bst + c] - Gb[m * bst + c]);
                    lv = fmaf(Rb[l * bst + c], w, lv);
                    av = fmaf(Qb[l * bst + c], w, av);
                }
                if (cb) {
                    lv += NT[l * C + m];
                    av += Am[l * C + m];
                }
                NT[l * C + m] = lv;  // the diagonal is overwritten below
                Am[l * C + m] = av;
            }
            if (CH) {  // decay the block in place: K<- (or E<-) and Q<-
                __syncthreads();
                for (int i = tid; i < C * kWideKB; i += kSimtThreads) {
                    const int l = i / kWideKB, c = i % kWideKB;
                    const float w = expf(Gb[l * bst + c]);
                    Qb[l * bst + c] *= w;
                    if (DEC) Eb[l * bst + c] *= w;
                    else Kb[l * bst + c] *= w;
                }
                __syncthreads();
            }
#pragma unroll
            for (int i = 0; i < kWideRegs; ++i) {
                const int l = warp + (kSimtThreads / kSimtRows) * i;
                if (l < C) {
                    float pa = pacc[i], qa = qacc[i];
#pragma unroll 4
                    for (int c = 0; c < kWideKB; ++c) {
                        const float sv = Ss[lane * sst + cb + c];
                        pa = fmaf(Rb[l * bst + c], sv, pa);
                        qa = fmaf(Qb[l * bst + c], sv, qa);
                    }
                    pacc[i] = pa;
                    qacc[i] = qa;
                }
            }
            __syncthreads();  // the next block overwrites this one
        }
        // ---- finish L -> N = diag(beta) L and A; P = V - K<- S^T ----
        for (int p = tid; p < npairs; p += kSimtThreads) {
            int l, m;
            tri_index(p, l, m);
            const float w = CH ? 1.f : expf(Gs[l] - Gs[m]);
            NT[l * C + m] = (m < l) ? bt[l] * NT[l * C + m] * w : 0.f;
            Am[l * C + m] *= w;
        }
#pragma unroll
        for (int i = 0; i < kWideRegs; ++i) {
            const int l = warp + (kSimtThreads / kSimtRows) * i;
            if (l < C) {
                float pv = 0.f;
                if (lane < nr && l < len) {
                    const float dl = CH ? 1.f : expf(Gs[l]);
                    const size_t vo = ((size_t)(c0 + l) * H + h) * dv + r0 + lane;
                    pv = (DEC ? ld_in(v, vo) * wg[vo] : ld_in(v, vo)) - dl * pacc[i];
                    qacc[i] *= dl;
                }
                Pm[l * kSimtRows + lane] = pv;
            }
        }
        __syncthreads();
        // ---- T: (I + N) T = diag(beta); T[i][j] (i > j) goes to NT[j][i] ----
        for (int j = tid; j < C; j += kSimtThreads) {
            const float bj = bt[j];
            for (int i = j + 1; i < C; ++i) {
                float acc = -NT[i * C + j] * bj;
                for (int m = j + 1; m < i; ++m) acc = fmaf(-NT[i * C + m], NT[j * C + m], acc);
                NT[j * C + i] = acc;
            }
        }
        __syncthreads();
        // ---- Z = T P ----
#pragma unroll
        for (int i = 0; i < kWideRegs; ++i) {
            const int l = warp + (kSimtThreads / kSimtRows) * i;
            if (l < C) {
                float z = bt[l] * Pm[l * kSimtRows + lane];
                for (int m = 0; m < l; ++m) z = fmaf(NT[m * C + l], Pm[m * kSimtRows + lane], z);
                Zm[l * kSimtRows + lane] = z;
            }
        }
        __syncthreads();
        // ---- O = Q<- S^T + A Z ----
#pragma unroll
        for (int i = 0; i < kWideRegs; ++i) {
            const int l = warp + (kSimtThreads / kSimtRows) * i;
            if (l < len && lane < nr) {
                float o = qacc[i];
                for (int m = 0; m <= l; ++m) o = fmaf(Am[l * C + m], Zm[m * kSimtRows + lane], o);
                st_out(out, ((size_t)(c0 + l) * H + h) * dv + r0 + lane, o);
            }
        }
        // ---- pass 2: S <- S Diag(exp(G_C)) + Z^T K-> ----
        for (int cb = 0; cb < dk; cb += kWideKB) {
            __syncthreads();  // Kb / Gb free
            load_block(c0, len, cb, false);
            for (int i = tid; i < C * kWideKB; i += kSimtThreads) {
                const int l = i / kWideKB, c = i % kWideKB;
                const float gap = CH ? Gb[(C - 1) * bst + c] - Gb[l * bst + c] : Gs[C - 1] - Gs[l];
                Kb[l * bst + c] *= expf(gap);
            }
            __syncthreads();
            for (int i = tid; i < kSimtRows * kWideKB; i += kSimtThreads) {
                const int r = i / kWideKB, c = i % kWideKB;
                const float gC = CH ? Gb[(C - 1) * bst + c] : Gs[C - 1];
                float acc = Ss[r * sst + cb + c] * expf(gC);
                for (int l = 0; l < C; ++l) acc = fmaf(Zm[l * kSimtRows + r], Kb[l * bst + c], acc);
                Ss[r * sst + cb + c] = acc;
            }
        }
    }
    __syncthreads();
    if (S_final) {
        for (int e = tid; e < nr * dk; e += kSimtThreads) {
            const int r = e / dk, c = e % dk;
            S_final[soff + (size_t)(r0 + r) * dk + c] = Ss[r * sst + c];
        }
    }
}

}  // namespace gdr

using namespace gdr;

namespace gdr_host {

static constexpr size_t kSimtSmemCap = 227u * 1024u;

// The resident layout where it fits, else the channel-blocked one.
static bool simt_wide(int C, int dk, bool channel, bool dec) {
    return sizeof(float) * (size_t)simt_layout(C, dk, channel, dec).total > kSimtSmemCap;
}

size_t simt_smem_bytes(int C, int dk, bool channel, bool dec) {
    if (!simt_wide(C, dk, channel, dec))
        return sizeof(float) * (size_t)simt_layout(C, dk, channel, dec).total;
    if (C > kWideMaxC || dk % kWideKB) return SIZE_MAX;
    return sizeof(float) * (size_t)wide_layout(C, dk, channel, dec).total;
}

template <typename Tin, bool CH, bool DEC = false>
static cudaError_t launch_simt(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *S0, void *out, float *S_final,
                               int T, int H, int dk, int dv, int C, const int32_t *cu, int n_seq,
                               int T_total, cudaStream_t st, const float *eg = nullptr,
                               const float *wg = nullptr) {
    const size_t smem = simt_smem_bytes(C, dk, CH, DEC);
    const bool wide = simt_wide(C, dk, CH, DEC);
    auto kern = wide ? fwd_simt_wide_kernel<Tin, CH, DEC> : fwd_simt_kernel<Tin, CH, DEC>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(n_seq * H), (unsigned)((dv + kSimtRows - 1) / kSimtRows));
    kern<<<grid, kSimtThreads, smem, st>>>(
        (const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta, eg, wg, S0, (Tin *)out, S_final,
        T, H, dk, dv, C, cu, T_total, n_seq, kChecked ? device_error_word() : nullptr);
    return cudaGetLastError();
}

// Gated DeltaNet-2: erase gate eg [.., d_k], write gate wg [.., d_v] instead of beta.
cudaError_t fwd_simt_gdn2_dispatch(const void *q, const void *k, const void *v, const float *g,
                                   const float *eg, const float *wg, const float *S0, void *out,
                                   float *S_final, int T, int H, int dk, int dv, int C,
                                   const int32_t *cu, int n_seq, int T_total, gdr_dtype dtype,
                                   gdr_gate gate, cudaStream_t st) {
    const bool ch = gate == GDR_GATE_PER_KEY_CHANNEL;
    if (dtype == GDR_BF16)
        return ch ? launch_simt<__nv_bfloat16, true, true>(q, k, v, g, nullptr, S0, out, S_final,
                                                           T, H, dk, dv, C, cu, n_seq, T_total,
                                                           st, eg, wg)
                  : launch_simt<__nv_bfloat16, false, true>(q, k, v, g, nullptr, S0, out, S_final,
                                                            T, H, dk, dv, C, cu, n_seq, T_total,
                                                            st, eg, wg);
    return ch ? launch_simt<float, true, true>(q, k, v, g, nullptr, S0, out, S_final, T, H, dk,
                                               dv, C, cu, n_seq, T_total, st, eg, wg)
              : launch_simt<float, false, true>(q, k, v, g, nullptr, S0, out, S_final, T, H, dk,
                                                dv, C, cu, n_seq, T_total, st, eg, wg);
}

cudaError_t fwd_simt_dispatch(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *S0, void *out, float *S_final,
                              int T, int H, int dk, int dv, int C, const int32_t *cu, int n_seq,
                              int T_total, gdr_dtype dtype, gdr_gate gate, cudaStream_t st) {
    const bool ch = gate == GDR_GATE_PER_KEY_CHANNEL;
    if (dtype == GDR_BF16)
        return ch ? launch_simt<__nv_bfloat16, true>(q, k, v, g, beta, S0, out, S_final, T, H, dk,
                                                     dv, C, cu, n_seq, T_total, st)
                  : launch_simt<__nv_bfloat16, false>(q, k, v, g, beta, S0, out, S_final, T, H,
                                                      dk, dv, C, cu, n_seq, T_total, st);
    return ch ? launch_simt<float, true>(q, k, v, g, beta, S0, out, S_final, T, H, dk, dv, C, cu,
                                         n_seq, T_total, st)
              : launch_simt<float, false>(q, k, v, g, beta, S0, out, S_final, T, H, dk, dv, C, cu,
                                          n_seq, T_total, st);
}

}  // namespace gdr_host
