// kla_chunk_simt.cu -- chunkwise KLA forward and backward on CUDA cores (fp32 arithmetic).
//
// This is the exact-precision path: every product is an fp32 FMA, so fp32 inputs keep
// ~1e-6 relative accuracy.  It serves fp32 inputs and every backward call; bf16 forward
// calls with Dk == Dv == 128 go to the tensor-core kernel instead.
//
// Chunkwise form ("Kaczmarz Linear Attention", section 4, Propositions 3-4, Eqs. 7-9),
// written on unit keys.  With k_i = r_i khat_i, the Kaczmarz write beta k e^T equals
// b khat (v/r - Sbar^T khat)^T with b = eta r^2/(r^2+eps) in [0, 1) and c = eta r/(r^2+eps)
// (the coefficient substitution of Appendix B.4 read on normalised keys).  The chunk system
// is then the GDN system on khat, which is well conditioned whatever the key norms:
//   G_i  = sum_{r<=i} g_r (inside the chunk), gamma_i = e^{G_i}, Gam_ij = e^{G_i - G_j}
//   L    = Diag(b) (Gam^- o Khat Khat^T)                       (strictly lower)
//   (I + L) U = Diag(c) V - Diag(b gamma) Khat S                 (Eq. 7)
//   O    = Diag(gamma) Q S + (Gam o Q Khat^T) U                  (Eq. 8)
//   S'   = gamma_last S + Khat^T Diag(e^{G_last - G}) U          (Eq. 9)
// Columns of V, U, O, S are independent (each state column evolves on its own), so a CTA
// owns one slice of NV value columns of one (b, h) and walks the chunks in order.
#include "kla_device.cuh"
#include "kla_launch.h"
#include "kla_tc_common.cuh"

namespace kla {
namespace {

constexpr int C = kChunk;
constexpr int NT = 256;

__device__ __forceinline__ size_t tok_index(int b, int t, int h, int T, int H) {
    return ((size_t)b * T + t) * H + h;
}

// acc[m][n] += sum_{kk<K} A(r0 + m*RS, kk) * B(kk, c0 + n*CS)
template <int K, int TM, int TN, int RS, int CS, typename FA, typename FB>
__device__ __forceinline__ void gemm_acc(float (&acc)[TM][TN], int r0, int c0, FA A, FB B) {
#pragma unroll 4
    for (int kk = 0; kk < K; ++kk) {
        float av[TM], bv[TN];
#pragma unroll
        for (int m = 0; m < TM; ++m) av[m] = A(r0 + m * RS, kk);
#pragma unroll
        for (int n = 0; n < TN; ++n) bv[n] = B(kk, c0 + n * CS);
#pragma unroll
        for (int m = 0; m < TM; ++m)
#pragma unroll
            for (int n = 0; n < TN; ++n) acc[m][n] = fmaf(av[m], bv[n], acc[m][n]);
    }
}

template <int TM, int TN>
__device__ __forceinline__ void zero(float (&acc)[TM][TN]) {
#pragma unroll
    for (int m = 0; m < TM; ++m)
#pragma unroll
        for (int n = 0; n < TN; ++n) acc[m][n] = 0.f;
}

// Load one chunk's keys (normalised) and queries, and the per-token coefficients.
// One warp per row; rows i >= n are zero-filled (they then contribute nothing).
template <int DK, typename Tin>
__device__ __forceinline__ void load_qk_rows(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                             const float* __restrict__ eta,
                                             const float* __restrict__ g, float eps, int b, int h,
                                             int t0, int n, int T, int H, float* Ks, float* Qs,
                                             int ldk, float* graw, float* bs, float* cs,
                                             float* us = nullptr) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int PER = DK / 32;
    for (int i = warp; i < C; i += NT / 32) {
        if (i < n) {
            const size_t ti = tok_index(b, t0 + i, h, T, H);
            const Tin* kr = k + ti * DK;
            const Tin* qr = q + ti * DK;
            float kv[PER];
            float r2 = 0.f;
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                kv[u] = to_f32(kr[lane + 32 * u]);
                r2 = fmaf(kv[u], kv[u], r2);
            }
            r2 = warp_sum(r2);
            const KaczCoef cf = kacz_coef(eta[ti], r2, eps);
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                Ks[i * ldk + lane + 32 * u] = kv[u] * cf.inv_r;
                Qs[i * ldk + lane + 32 * u] = to_f32(qr[lane + 32 * u]);
            }
            if (lane == 0) {
                graw[i] = g[ti];
                bs[i] = cf.b;
                cs[i] = cf.c;
                // value coefficient of U for the backward: c, except at a key of zero norm,
                // where U's row takes beta v (it meets only khat = 0 there, but row i of dkhat
                // then equals the exact dk = beta Gbar v)
                if (us) us[i] = r2 == 0.f ? (eps < 0.f ? eta[ti] : (eps > 0.f ? eta[ti] / eps : 0.f)) : cf.c;
            }
        } else {
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                Ks[i * ldk + lane + 32 * u] = 0.f;
                Qs[i * ldk + lane + 32 * u] = 0.f;
            }
            if (lane == 0) {
                graw[i] = 0.f;
                bs[i] = 0.f;
                cs[i] = 0.f;
                if (us) us[i] = 0.f;
            }
        }
    }
}

// Inclusive prefix sum of the log-decays inside the chunk, then the decay factors.
__device__ __forceinline__ void chunk_decay(const float* graw, float* Gs, float* gams, float* dels,
                                            int n) {
    if (threadIdx.x == 0) {
        float acc = 0.f;
        for (int i = 0; i < C; ++i) {
            acc += graw[i];
            Gs[i] = acc;
        }
    }
    __syncthreads();
    if (threadIdx.x < C) {
        const int i = threadIdx.x;
        gams[i] = expf(Gs[i]);
        dels[i] = expf(Gs[n - 1] - Gs[i]);
    }
}

// ------------------------------------------------------------------------------------
// Forward
// ------------------------------------------------------------------------------------
template <int DK, typename Tin, typename TOut>
__global__ void __launch_bounds__(NT, 1) chunk_fwd_simt_kernel(FwdArgs a) {
    constexpr int NV = 64;
    constexpr int LDK = DK + 1, LDV = NV + 1, LDC = C + 1;
    constexpr int TMS = DK / 16;  // state rows per thread in the state update
    extern __shared__ float sm[];
    float* Ks = sm;              // C x LDK   unit keys
    float* Qs = Ks + C * LDK;    // C x LDK
    float* Rs = Qs + C * LDK;    // C x LDV   c V -> R -> U
    float* Xs = Rs + C * LDV;    // C x LDV   Khat S
    float* Ss = Xs + C * LDV;    // DK x LDV  state slice
    float* Lm = Ss + DK * LDV;   // C x LDC   L (strictly lower)
    float* Pm = Lm + C * LDC;    // C x LDC   Gam o Q Khat^T (lower incl. diagonal)
    float* Gs = Pm + C * LDC;
    float* bs = Gs + C;
    float* cs = bs + C;
    float* gams = cs + C;
    float* dels = gams + C;
    float* graw = dels + C;

    const int v0 = blockIdx.x * NV, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tx = tid & 15, ty = tid >> 4;
    const int T = a.T, H = a.H, Dv = a.Dv;
    const Tin* q = static_cast<const Tin*>(a.q);
    const Tin* k = static_cast<const Tin*>(a.k);
    const Tin* v = static_cast<const Tin*>(a.v);
    TOut* o = static_cast<TOut*>(a.o);
    const size_t sbase = ((size_t)b * H + h) * DK * Dv;
    const int NC = (T + C - 1) / C;

    for (int x = tid; x < DK * NV; x += NT) {
        const int r = x / NV, c = x % NV;
        Ss[r * LDV + c] = a.S0 ? a.S0[sbase + (size_t)r * Dv + v0 + c] : 0.f;
    }

    for (int ci = 0; ci < NC; ++ci) {
        const int t0 = ci * C;
        const int n = min(C, T - t0);
        __syncthreads();
        if (a.S_chunks) {
            float* dst = a.S_chunks + (((size_t)b * H + h) * NC + ci) * DK * Dv;
            for (int x = tid; x < DK * NV; x += NT) {
                const int r = x / NV, c = x % NV;
                dst[(size_t)r * Dv + v0 + c] = Ss[r * LDV + c];
            }
        }
        load_qk_rows<DK, Tin>(q, k, a.eta, a.g, a.eps, b, h, t0, n, T, H, Ks, Qs, LDK, graw, bs, cs);
        __syncthreads();
        // c V into Rs (one warp per row, NV = 64 columns = 2 per lane)
        for (int i = warp; i < C; i += NT / 32) {
            for (int j = lane; j < NV; j += 32) {
                float val = 0.f;
                if (i < n) val = cs[i] * to_f32(v[tok_index(b, t0 + i, h, T, H) * Dv + v0 + j]);
                Rs[i * LDV + j] = val;
            }
        }
        chunk_decay(graw, Gs, gams, dels, n);
        __syncthreads();

        // Gram matrices: L = Diag(b)(Gam^- o Khat Khat^T), P = Gam o Q Khat^T
        {
            float akk[4][4], aqk[4][4];
            zero(akk);
            zero(aqk);
            auto Bk = [&](int d, int j) { return Ks[j * LDK + d]; };
            gemm_acc<DK, 4, 4, 16, 16>(akk, ty, tx, [&](int i, int d) { return Ks[i * LDK + d]; }, Bk);
            gemm_acc<DK, 4, 4, 16, 16>(aqk, ty, tx, [&](int i, int d) { return Qs[i * LDK + d]; }, Bk);
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) {
                    const int i = ty + 16 * m, j = tx + 16 * nn;
                    const float gij = (j <= i) ? expf(Gs[i] - Gs[j]) : 0.f;
                    Lm[i * LDC + j] = (j < i) ? bs[i] * gij * akk[m][nn] : 0.f;
                    Pm[i * LDC + j] = gij * aqk[m][nn];
                }
        }
        // X = Khat S
        {
            float ax[4][4];
            zero(ax);
            gemm_acc<DK, 4, 4, 16, 16>(ax, ty, tx, [&](int i, int d) { return Ks[i * LDK + d]; },
                                       [&](int d, int j) { return Ss[d * LDV + j]; });
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) Xs[(ty + 16 * m) * LDV + tx + 16 * nn] = ax[m][nn];
        }
        __syncthreads();
        // R = c V - Diag(b gamma) Khat S
        for (int x = tid; x < C * NV; x += NT) {
            const int i = x / NV, j = x % NV;
            Rs[i * LDV + j] -= bs[i] * gams[i] * Xs[i * LDV + j];
        }
        __syncthreads();
        // Forward substitution (I + L) U = R, row by row (Appendix B.2).
        {
            const int col = tid >> 2, part = tid & 3;
            for (int i = 1; i < n; ++i) {
                float s = 0.f;
                for (int j = part; j < i; j += 4) s = fmaf(Lm[i * LDC + j], Rs[j * LDV + col], s);
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                if (part == 0) Rs[i * LDV + col] -= s;
                __syncthreads();
            }
        }
        // O = Diag(gamma) Q S + P U
        if (o != nullptr) {
            float ao[4][4], ap[4][4];
            zero(ao);
            zero(ap);
            gemm_acc<DK, 4, 4, 16, 16>(ao, ty, tx, [&](int i, int d) { return Qs[i * LDK + d]; },
                                       [&](int d, int j) { return Ss[d * LDV + j]; });
            gemm_acc<C, 4, 4, 16, 16>(ap, ty, tx, [&](int i, int t) { return Pm[i * LDC + t]; },
                                      [&](int t, int j) { return Rs[t * LDV + j]; });
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = ty + 16 * m;
                if (i < n) {
                    TOut* orow = o + tok_index(b, t0 + i, h, T, H) * Dv + v0;
#pragma unroll
                    for (int nn = 0; nn < 4; ++nn)
                        orow[tx + 16 * nn] = from_f32<TOut>(fmaf(gams[i], ao[m][nn], ap[m][nn]));
                }
            }
        }
        // S' = gamma_last S + Khat^T Diag(delta) U
        {
            float as[TMS][4];
            zero(as);
            gemm_acc<C, TMS, 4, 16, 16>(as, ty, tx, [&](int r, int t) { return Ks[t * LDK + r]; },
                                        [&](int t, int j) { return dels[t] * Rs[t * LDV + j]; });
            const float gC = gams[n - 1];
            __syncthreads();
#pragma unroll
            for (int m = 0; m < TMS; ++m)
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) {
                    float* sp = &Ss[(ty + 16 * m) * LDV + tx + 16 * nn];
                    *sp = fmaf(gC, *sp, as[m][nn]);
                }
        }
    }
    __syncthreads();
    if (a.S_T) {
        for (int x = tid; x < DK * NV; x += NT) {
            const int r = x / NV, c = x % NV;
            a.S_T[sbase + (size_t)r * Dv + v0 + c] = Ss[r * LDV + c];
        }
    }
}

template <int DK>
constexpr size_t fwd_smem_bytes() {
    return sizeof(float) * (2 * C * (DK + 1) + 2 * C * 65 + DK * 65 + 2 * C * (C + 1) + 6 * C);
}

// ------------------------------------------------------------------------------------
// Backward
//
// Per chunk (newest first) with incoming state S (from S_chunks) and dS' the gradient
// w.r.t. the chunk's outgoing state:
//   dU  = (Gam o Q Khat^T)^T dO + Diag(delta) Khat dS'
//   dR  = (I + L)^{-T} dU = T^T dU,  T = (I + L)^{-1} inverted once per chunk (doubling)
//   dS  = gamma_last dS' + Q^T Diag(gamma) dO - Khat^T Diag(b gamma) dR   (carried on)
//   dV  = Diag(c) dR,  dc_i = dR_i . v_i
//   D   = -dR U^T (strictly lower) -> db_i += sum_t D_it (Gam o KK)_it,
//         E = D o Diag(b) Gam,  dKhat += E Khat + E^T Khat
//   Y   = dO U^T (lower) -> F = Y o Gam,  dQ += F Khat,  dKhat += F^T Q
//   dQ += Diag(gamma) dO S^T;  dKhat += -Diag(b gamma) dR S^T + Diag(delta) U dS'^T
//   db_i += -gamma_i dR_i.(Khat S)_i;  dgamma_i = -b_i dR_i.(Khat S)_i + dO_i.(Q S)_i
//   ddelta_i = U_i.(Khat dS')_i;  dgamma_last = <dS', S>
//   dG from every decay factor, then dg = reverse cumulative sum inside the chunk.
// A CTA owns NV = 32 value columns; the column-coupled gradients (dq, dkhat, db, dc, dG)
// are partial sums over its columns and are added atomically into fp32 accumulators.
// ------------------------------------------------------------------------------------
template <int DK, typename Tin, typename TOut>
__global__ void __launch_bounds__(NT, 1) chunk_bwd_simt_kernel(BwdArgs a) {
    constexpr int NV = 32;
    constexpr int LDK = DK + 1, LDV = NV + 1, LDC = C + 1;
    constexpr int TMK = DK / 16;  // state rows per thread for DK x NV outputs
    constexpr int TNK = DK / 16;  // key columns per thread for C x DK outputs
    extern __shared__ float sm[];
    float* Ks = sm;               // C x LDK
    float* Qs = Ks + C * LDK;     // C x LDK
    float* Ss = Qs + C * LDK;     // DK x LDV  incoming state slice
    float* dSs = Ss + DK * LDV;   // DK x LDV  gradient w.r.t. outgoing state slice
    float* Us = dSs + DK * LDV;   // C x LDV   cV -> R -> U
    float* dRs = Us + C * LDV;    // C x LDV   dU -> dR
    float* dOs = dRs + C * LDV;   // C x LDV
    float* Xs = dOs + C * LDV;    // C x LDV   Khat S
    float* QSs = Xs + C * LDV;    // C x LDV   Q S
    float* KdS = QSs + C * LDV;   // C x LDV   Khat dS'
    float* Lh = KdS + C * LDV;    // C x LDC   Gam o Khat Khat^T (strict), later E
    float* Pm = Lh + C * LDC;     // C x LDC   Gam o Q Khat^T (incl. diag), later F
    float* Gs = Pm + C * LDC;
    float* bs = Gs + C;
    float* cs = bs + C;
    float* gams = cs + C;
    float* dels = gams + C;
    float* graw = dels + C;
    float* dGs = graw + C;
    float* dbs = dGs + C;
    float* dcs = dbs + C;
    float* red = dcs + C;  // 8
    float* Tf = red + 8;                // C x tcc::LDL   T = (I + L)^{-1}  (16-byte aligned)
    float* ucs = Tf + C * tcc::LDL + 1024 + C * LDV;  // C   value coefficient of U
    float* Xinv = Tf + C * tcc::LDL;    // 1024           scratch of the inverse
    float* Tmp = Xinv + 1024;           // C x LDV        U = T R and dR = T^T dU before copy-back

    const int v0 = blockIdx.x * NV, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tx = tid & 15, ty = tid >> 4;
    const int T = a.T, H = a.H, Dv = a.Dv;
    const Tin* q = static_cast<const Tin*>(a.q);
    const Tin* k = static_cast<const Tin*>(a.k);
    const Tin* v = static_cast<const Tin*>(a.v);
    const Tin* dO = static_cast<const Tin*>(a.dO);
    TOut* dv = static_cast<TOut*>(a.dv);
    const size_t sbase = ((size_t)b * H + h) * DK * Dv;
    const int NC = (T + C - 1) / C;

    for (int x = tid; x < DK * NV; x += NT) {
        const int r = x / NV, c = x % NV;
        dSs[r * LDV + c] = a.dS_T ? a.dS_T[sbase + (size_t)r * Dv + v0 + c] : 0.f;
    }

    for (int ci = NC - 1; ci >= 0; --ci) {
        const int t0 = ci * C;
        const int n = min(C, T - t0);
        __syncthreads();
        load_qk_rows<DK, Tin>(q, k, a.eta, a.g, a.eps, b, h, t0, n, T, H, Ks, Qs, LDK, graw, bs, cs, ucs);
        {
            const float* src = a.S_chunks + (((size_t)b * H + h) * NC + ci) * DK * Dv;
            for (int x = tid; x < DK * NV; x += NT) {
                const int r = x / NV, c = x % NV;
                Ss[r * LDV + c] = src[(size_t)r * Dv + v0 + c];
            }
        }
        if (tid < C) {
            dGs[tid] = 0.f;
            dbs[tid] = 0.f;
            dcs[tid] = 0.f;
        }
        __syncthreads();
        for (int i = warp; i < C; i += NT / 32) {  // NV == 32: one column per lane
            float cv = 0.f, dov = 0.f;
            if (i < n) {
                const size_t ti = tok_index(b, t0 + i, h, T, H);
                cv = ucs[i] * to_f32(v[ti * Dv + v0 + lane]);
                dov = to_f32(dO[ti * Dv + v0 + lane]);
            }
            Us[i * LDV + lane] = cv;
            dOs[i * LDV + lane] = dov;
        }
        chunk_decay(graw, Gs, gams, dels, n);
        __syncthreads();

        // Gram matrices (without b): Lh = Gam^- o KK^T, Pm = Gam o Q Khat^T
        {
            float akk[4][4], aqk[4][4];
            zero(akk);
            zero(aqk);
            auto Bk = [&](int d, int j) { return Ks[j * LDK + d]; };
            gemm_acc<DK, 4, 4, 16, 16>(akk, ty, tx, [&](int i, int d) { return Ks[i * LDK + d]; }, Bk);
            gemm_acc<DK, 4, 4, 16, 16>(aqk, ty, tx, [&](int i, int d) { return Qs[i * LDK + d]; }, Bk);
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) {
                    const int i = ty + 16 * m, j = tx + 16 * nn;
                    const float gij = (j <= i) ? expf(Gs[i] - Gs[j]) : 0.f;
                    Lh[i * LDC + j] = (j < i) ? gij * akk[m][nn] : 0.f;
                    Pm[i * LDC + j] = gij * aqk[m][nn];
                }
        }
        // X = Khat S, QS = Q S, KdS = Khat dS'   (C x NV each)
        {
            float ax[4][2], aq[4][2], ad[4][2];
            zero(ax);
            zero(aq);
            zero(ad);
            gemm_acc<DK, 4, 2, 16, 16>(ax, ty, tx, [&](int i, int d) { return Ks[i * LDK + d]; },
                                       [&](int d, int j) { return Ss[d * LDV + j]; });
            gemm_acc<DK, 4, 2, 16, 16>(aq, ty, tx, [&](int i, int d) { return Qs[i * LDK + d]; },
                                       [&](int d, int j) { return Ss[d * LDV + j]; });
            gemm_acc<DK, 4, 2, 16, 16>(ad, ty, tx, [&](int i, int d) { return Ks[i * LDK + d]; },
                                       [&](int d, int j) { return dSs[d * LDV + j]; });
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int nn = 0; nn < 2; ++nn) {
                    const int i = ty + 16 * m, j = tx + 16 * nn;
                    Xs[i * LDV + j] = ax[m][nn];
                    QSs[i * LDV + j] = aq[m][nn];
                    KdS[i * LDV + j] = ad[m][nn];
                }
        }
        __syncthreads();
        for (int x = tid; x < C * NV; x += NT) {
            const int i = x / NV, j = x % NV;
            Us[i * LDV + j] -= bs[i] * gams[i] * Xs[i * LDV + j];
        }
        __syncthreads();
        // T = (I + Diag(b) Lh)^{-1} (Lh is zero on and above the diagonal; rows past the last
        // token are unit rows), then U = T R
        for (int x = tid; x < C * C; x += NT) {
            const int i = x / C, j = x % C;
            Tf[i * tcc::LDL + j] = bs[i] * Lh[i * LDC + j];
        }
        __syncthreads();
        tcc::invert_unit_lower64_doubling<NT>(Tf, Xinv, tid);
        {
            float au[4][2];
            zero(au);
            gemm_acc<C, 4, 2, 16, 16>(au, ty, tx, [&](int i, int j) { return Tf[i * tcc::LDL + j]; },
                                      [&](int j, int c) { return Us[j * LDV + c]; });
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int nn = 0; nn < 2; ++nn) Tmp[(ty + 16 * m) * LDV + tx + 16 * nn] = au[m][nn];
            __syncthreads();
            for (int x = tid; x < C * NV; x += NT) Us[(x / NV) * LDV + x % NV] = Tmp[(x / NV) * LDV + x % NV];
            __syncthreads();
        }
        // dU = P^T dO + Diag(delta) Khat dS'
        {
            float au[4][2];
            zero(au);
            gemm_acc<C, 4, 2, 16, 16>(au, ty, tx, [&](int i, int t) { return Pm[t * LDC + i]; },
                                      [&](int t, int j) { return dOs[t * LDV + j]; });
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int nn = 0; nn < 2; ++nn) {
                    const int i = ty + 16 * m, j = tx + 16 * nn;
                    dRs[i * LDV + j] = au[m][nn] + dels[i] * KdS[i * LDV + j];
                }
        }
        __syncthreads();
        // dR = T^T dU
        {
            float ar[4][2];
            zero(ar);
            gemm_acc<C, 4, 2, 16, 16>(ar, ty, tx, [&](int i, int j) { return Tf[j * tcc::LDL + i]; },
                                      [&](int j, int c) { return dRs[j * LDV + c]; });
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int nn = 0; nn < 2; ++nn) Tmp[(ty + 16 * m) * LDV + tx + 16 * nn] = ar[m][nn];
            __syncthreads();
            for (int x = tid; x < C * NV; x += NT) dRs[(x / NV) * LDV + x % NV] = Tmp[(x / NV) * LDV + x % NV];
            __syncthreads();
        }
        // Row scalars (one warp per row, one column per lane) and dv.
        for (int i = warp; i < n; i += NT / 32) {
            const size_t ti = tok_index(b, t0 + i, h, T, H);
            const float dr = dRs[i * LDV + lane];
            const float vv = to_f32(v[ti * Dv + v0 + lane]);
            dv[ti * Dv + v0 + lane] = from_f32<TOut>(cs[i] * dr);
            const float s_rv = warp_sum(dr * vv);
            const float s_rx = warp_sum(dr * Xs[i * LDV + lane]);
            const float s_oq = warp_sum(dOs[i * LDV + lane] * QSs[i * LDV + lane]);
            const float s_uk = warp_sum(Us[i * LDV + lane] * KdS[i * LDV + lane]);
            if (lane == 0) {
                atomicAdd(&dcs[i], s_rv);
                atomicAdd(&dbs[i], -gams[i] * s_rx);
                const float dgam = -bs[i] * s_rx + s_oq;
                atomicAdd(&dGs[i], gams[i] * dgam - dels[i] * s_uk);
                atomicAdd(&dGs[n - 1], dels[i] * s_uk);
            }
        }
        // <dS', S> for the outgoing decay gamma_last
        {
            float p = 0.f;
            for (int x = tid; x < DK * NV; x += NT) {
                const int r = x / NV, c = x % NV;
                p = fmaf(dSs[r * LDV + c], Ss[r * LDV + c], p);
            }
            p = warp_sum(p);
            if (lane == 0) red[warp] = p;
        }
        __syncthreads();
        if (tid == 0) {
            float p = 0.f;
            for (int w = 0; w < NT / 32; ++w) p += red[w];
            atomicAdd(&dGs[n - 1], gams[n - 1] * p);
        }
        // Y = dO U^T and D = -dR U^T (C x C); transform in place into F (Pm) and E (Lh).
        {
            float ay[4][4], ad[4][4];
            zero(ay);
            zero(ad);
            auto Bu = [&](int j, int t) { return Us[t * LDV + j]; };
            gemm_acc<NV, 4, 4, 16, 16>(ay, ty, tx, [&](int i, int j) { return dOs[i * LDV + j]; }, Bu);
            gemm_acc<NV, 4, 4, 16, 16>(ad, ty, tx, [&](int i, int j) { return dRs[i * LDV + j]; }, Bu);
            float rowG[4] = {0.f, 0.f, 0.f, 0.f}, rowB[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = ty + 16 * m;
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) {
                    const int t = tx + 16 * nn;
                    const float Dv_ = -ad[m][nn];
                    const float gij = (t <= i) ? expf(Gs[i] - Gs[t]) : 0.f;
                    const float pm = Pm[i * LDC + t];
                    const float lh = Lh[i * LDC + t];
                    const float F = ay[m][nn] * gij;                      // zero above diagonal
                    const float dgg_o = ay[m][nn] * pm;                   // Y o Gam o QK
                    const float E = (t < i) ? Dv_ * bs[i] * gij : 0.f;
                    const float dgg_l = (t < i) ? Dv_ * bs[i] * lh : 0.f;
                    rowB[m] += (t < i) ? Dv_ * lh : 0.f;
                    const float dgg = dgg_o + dgg_l;
                    rowG[m] += dgg;
                    if (dgg != 0.f) atomicAdd(&dGs[t], -dgg);
                    Pm[i * LDC + t] = F;
                    Lh[i * LDC + t] = E;
                }
                atomicAdd(&dGs[i], rowG[m]);
                atomicAdd(&dbs[i], rowB[m]);
            }
        }
        __syncthreads();
        // dq and dkhat partials, C x DK:
        //   dq    = Diag(gamma) dO S^T + F Khat
        //   dkhat = -Diag(b gamma) dR S^T + Diag(delta) U dS'^T + F^T Q + (E + E^T) Khat
        {
            float aq[4][TNK], ak[4][TNK];
            zero(aq);
            zero(ak);
            float rg[4], rbg[4], rd[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = ty + 16 * m;
                rg[m] = gams[i];
                rbg[m] = -bs[i] * gams[i];
                rd[m] = dels[i];
            }
#pragma unroll 2
            for (int j = 0; j < NV; ++j) {
                float a1[4], a2[4], a3[4], b1[TNK], b2[TNK];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int i = ty + 16 * m;
                    a1[m] = rg[m] * dOs[i * LDV + j];
                    a2[m] = rbg[m] * dRs[i * LDV + j];
                    a3[m] = rd[m] * Us[i * LDV + j];
                }
#pragma unroll
                for (int nn = 0; nn < TNK; ++nn) {
                    const int r = tx + 16 * nn;
                    b1[nn] = Ss[r * LDV + j];
                    b2[nn] = dSs[r * LDV + j];
                }
#pragma unroll
                for (int m = 0; m < 4; ++m)
#pragma unroll
                    for (int nn = 0; nn < TNK; ++nn) {
                        aq[m][nn] = fmaf(a1[m], b1[nn], aq[m][nn]);
                        ak[m][nn] = fmaf(a2[m], b1[nn], fmaf(a3[m], b2[nn], ak[m][nn]));
                    }
            }
#pragma unroll 2
            for (int t = 0; t < C; ++t) {
                float f[4], ft[4], e[4], bk[TNK], bq[TNK];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int i = ty + 16 * m;
                    f[m] = Pm[i * LDC + t];
                    ft[m] = Pm[t * LDC + i];
                    e[m] = Lh[i * LDC + t] + Lh[t * LDC + i];
                }
#pragma unroll
                for (int nn = 0; nn < TNK; ++nn) {
                    const int r = tx + 16 * nn;
                    bk[nn] = Ks[t * LDK + r];
                    bq[nn] = Qs[t * LDK + r];
                }
#pragma unroll
                for (int m = 0; m < 4; ++m)
#pragma unroll
                    for (int nn = 0; nn < TNK; ++nn) {
                        aq[m][nn] = fmaf(f[m], bk[nn], aq[m][nn]);
                        ak[m][nn] = fmaf(ft[m], bq[nn], fmaf(e[m], bk[nn], ak[m][nn]));
                    }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = ty + 16 * m;
                if (i < n) {
                    const size_t ti = tok_index(b, t0 + i, h, T, H);
#pragma unroll
                    for (int nn = 0; nn < TNK; ++nn) {
                        const int r = tx + 16 * nn;
                        atomicAdd(&a.acc_dq[ti * DK + r], aq[m][nn]);
                        atomicAdd(&a.acc_dkh[ti * DK + r], ak[m][nn]);
                    }
                }
            }
        }
        // new dS' = gamma_last dS' + Q^T Diag(gamma) dO - Khat^T Diag(b gamma) dR
        {
            float as[TMK][2];
            zero(as);
            gemm_acc<C, TMK, 2, 16, 16>(as, ty, tx, [&](int r, int t) { return Qs[t * LDK + r]; },
                                        [&](int t, int j) { return gams[t] * dOs[t * LDV + j]; });
            gemm_acc<C, TMK, 2, 16, 16>(as, ty, tx, [&](int r, int t) { return Ks[t * LDK + r]; },
                                        [&](int t, int j) { return -bs[t] * gams[t] * dRs[t * LDV + j]; });
            const float gC = gams[n - 1];
            __syncthreads();
#pragma unroll
            for (int m = 0; m < TMK; ++m)
#pragma unroll
                for (int nn = 0; nn < 2; ++nn) {
                    float* sp = &dSs[(ty + 16 * m) * LDV + tx + 16 * nn];
                    *sp = fmaf(gC, *sp, as[m][nn]);
                }
        }
        // scalar gradients of this chunk (all smem atomics above are complete)
        if (tid < n) {
            const size_t ti = tok_index(b, t0 + tid, h, T, H);
            atomicAdd(&a.acc_db[ti], dbs[tid]);
            atomicAdd(&a.acc_dc[ti], dcs[tid]);
            atomicAdd(&a.acc_dG[ti], dGs[tid]);
        }
    }
    __syncthreads();
    for (int x = tid; x < DK * NV; x += NT) {
        const int r = x / NV, c = x % NV;
        a.dS0[sbase + (size_t)r * Dv + v0 + c] = dSs[r * LDV + c];
    }
}

template <int DK>
constexpr size_t bwd_smem_bytes() {
    return sizeof(float) * (2 * C * (DK + 1) + 2 * DK * 33 + 6 * C * 33 + 2 * C * (C + 1) + 9 * C + 8 +
                            C * tcc::LDL + 1024 + C * 33 + C);
}

// dq to the output type; dk and deta from the unit-key gradients:
//   b = eta r^2/(r^2+eps), c = eta r/(r^2+eps), khat = k/r
//   deta = db r^2/den + dc r/den,  dr = db eta 2 r eps/den^2 + dc eta (eps - r^2)/den^2
//   dk   = (dkhat - khat (khat . dkhat)) / r + khat dr
// At a key of zero norm the accumulated dkhat already is dk (U's row there was beta v).
template <int DK, typename Tin, typename TOut>
__global__ void __launch_bounds__(256) bwd_finalize_kernel(BwdArgs a, size_t ntok) {
    const size_t w = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= ntok) return;
    constexpr int PER = DK / 32;
    const Tin* k = static_cast<const Tin*>(a.k);
    TOut* dq = static_cast<TOut*>(a.dq);
    TOut* dk = static_cast<TOut*>(a.dk);
    float kv[PER], dkh[PER];
    float r2 = 0.f;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        kv[u] = to_f32(k[w * DK + lane + 32 * u]);
        dkh[u] = a.acc_dkh[w * DK + lane + 32 * u];
        r2 = fmaf(kv[u], kv[u], r2);
        dq[w * DK + lane + 32 * u] = from_f32<TOut>(a.acc_dq[w * DK + lane + 32 * u]);
    }
    r2 = warp_sum(r2);
    const float r = sqrtf(r2);
    const float den = r2 + a.eps;
    const bool direct = a.eps < 0.f;  // beta = eta as given: b = eta r^2, c = eta r
    const bool live = (direct || den > 0.f) && r > 0.f;
    const float inv_r = live ? 1.f / r : 0.f;
    float kd = 0.f;
#pragma unroll
    for (int u = 0; u < PER; ++u) kd = fmaf(kv[u] * inv_r, dkh[u], kd);
    kd = warp_sum(kd);
    const float db = a.acc_db[w], dc = a.acc_dc[w], et = a.eta[w];
    float deta = 0.f, dr = 0.f;
    if (live && direct) {
        deta = db * r2 + dc * r;
        dr = db * et * 2.f * r + dc * et;
    } else if (live) {
        deta = db * r2 / den + dc * r / den;
        dr = (db * et * 2.f * r * a.eps + dc * et * (a.eps - r2)) / (den * den);
    }
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const float kh = kv[u] * inv_r;
        const float val = live ? (dkh[u] - kh * kd) * inv_r + kh * dr : dkh[u];
        dk[w * DK + lane + 32 * u] = from_f32<TOut>(val);
    }
    if (lane == 0) a.deta[w] = deta;
}

// dg_r = sum_{i >= r} dG_i inside each chunk (the log-decay enters only through G).
__global__ void bwd_dg_kernel(BwdArgs a) {
    const int NC = (a.T + C - 1) / C;
    const size_t id = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t total = (size_t)a.B * a.H * NC;
    if (id >= total) return;
    const int ci = (int)(id % NC);
    const int h = (int)((id / NC) % a.H);
    const int b = (int)(id / ((size_t)NC * a.H));
    const int t0 = ci * C;
    const int n = min(C, a.T - t0);
    float acc = 0.f;
    for (int i = n - 1; i >= 0; --i) {
        const size_t ti = tok_index(b, t0 + i, h, a.T, a.H);
        acc += a.acc_dG[ti];
        a.dg[ti] = acc;
    }
}

template <int DK, typename Tin, typename TOut>
cudaError_t fwd_launch_t(const FwdArgs& a, cudaStream_t st) {
    const size_t smem = fwd_smem_bytes<DK>();
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_simt_kernel<DK, Tin, TOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.Dv / 64, a.H, a.B);
    chunk_fwd_simt_kernel<DK, Tin, TOut><<<grid, NT, smem, st>>>(a);
    return cudaGetLastError();
}

template <int DK, typename Tin, typename TOut>
cudaError_t bwd_launch_t(const BwdArgs& a, cudaStream_t st) {
    const size_t smem = bwd_smem_bytes<DK>();
    cudaError_t e = cudaFuncSetAttribute(chunk_bwd_simt_kernel<DK, Tin, TOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.Dv / 32, a.H, a.B);
    chunk_bwd_simt_kernel<DK, Tin, TOut><<<grid, NT, smem, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t ntok = (size_t)a.B * a.T * a.H;
    if (ntok > 0) {
        bwd_finalize_kernel<DK, Tin, TOut><<<(unsigned)((ntok + 7) / 8), 256, 0, st>>>(a, ntok);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const size_t nch = (size_t)a.B * a.H * ((a.T + C - 1) / C);
        bwd_dg_kernel<<<(unsigned)((nch + 127) / 128), 128, 0, st>>>(a);
        e = cudaGetLastError();
    }
    return e;
}

template <int DK, typename Tin>
cudaError_t fwd_launch_o(const FwdArgs& a, cudaStream_t st) {
    return a.out_bf16 ? fwd_launch_t<DK, Tin, __nv_bfloat16>(a, st) : fwd_launch_t<DK, Tin, float>(a, st);
}

template <int DK, typename Tin>
cudaError_t bwd_launch_o(const BwdArgs& a, cudaStream_t st) {
    return a.out_bf16 ? bwd_launch_t<DK, Tin, __nv_bfloat16>(a, st) : bwd_launch_t<DK, Tin, float>(a, st);
}

}  // namespace

cudaError_t launch_chunk_fwd_simt(const FwdArgs& a, cudaStream_t st) {
    if (a.bf16) return a.Dk == 128 ? fwd_launch_o<128, __nv_bfloat16>(a, st)
                                   : fwd_launch_o<64, __nv_bfloat16>(a, st);
    return a.Dk == 128 ? fwd_launch_o<128, float>(a, st) : fwd_launch_o<64, float>(a, st);
}

cudaError_t launch_chunk_bwd_simt(const BwdArgs& a, cudaStream_t st) {
    if (a.bf16) return a.Dk == 128 ? bwd_launch_o<128, __nv_bfloat16>(a, st)
                                   : bwd_launch_o<64, __nv_bfloat16>(a, st);
    return a.Dk == 128 ? bwd_launch_o<128, float>(a, st) : bwd_launch_o<64, float>(a, st);
}

}  // namespace kla
