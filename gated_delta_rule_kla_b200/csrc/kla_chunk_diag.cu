// kla_chunk_diag.cu -- KLA with diagonal (per-key-channel) gating on CUDA cores (fp32).
//
// "Kaczmarz Linear Attention", Appendix A.5 (the Kaczmarz step is decay-agnostic) and B.5 (the
// chunk form under a diagonal decay): the decay of token t is Diag(alpha_t) with
// alpha_t = exp(g_t), g_t in R^{Dk} (one log-decay per key channel), so per head
//   Sbar = Diag(alpha_t) S_{t-1};  e_t = v_t - Sbar^T k_t;  S_t = Sbar + beta_t k_t e_t^T;
//   o_t = S_t^T q_t,  beta_t = eta_t / (||k_t||^2 + eps)  (or eta_t as given, direct mode).
//
// Chunk form on unit keys (k = r khat, b = eta r^2/(r^2+eps), c = eta r/(r^2+eps) as for scalar
// gating), with G_i = sum_{s<=i} g_s the per-channel log-decay inside the chunk and
// E_ij = exp(G_i - G_j) (a vector over channels, j <= i, every factor <= 1 for g <= 0):
//   L_ij = b_i sum_c khat_i[c] khat_j[c] E_ij[c]   (j < i)      P_ij = sum_c q_i[c] khat_j[c] E_ij[c]
//   (I + L) U = Diag(c) V - Diag(b) (Khat o Gam) S                 Gam_i = exp(G_i)
//   O = (Q o Gam) S + P U
//   S' = Diag(Gam_last) S + (Khat o Del)^T U                       Del_j = exp(G_last - G_j)
// Unlike scalar gating, the decay cannot be taken out of the channel sums, so the chunk's
// pairwise factors are formed channel by channel.  The kernels use 16-token chunks: every factor
// is then exp of a non-positive number (no rescaling reference that could overflow, whatever the
// decay), and the pairwise work per token stays small.
//
// Columns of V, U, O, S are independent, so a CTA owns NV value columns of one (b, h) and walks
// the chunks in order (forward) or newest first (backward, from the chunk-start states the
// forward kernel saved in the workspace).  The backward's column-coupled gradients (dq, dkhat,
// db, dc, dG per channel) are partial sums over a CTA's columns, added atomically into fp32
// accumulators; a finishing kernel maps (dkhat, db, dc) to (dk, deta) and the per-channel dG to
// dg by a reverse cumulative sum inside each 16-token chunk.
#include "kla_device.cuh"
#include "kla_launch.h"
#include "kla_sm100.cuh"

namespace kla {

__device__ unsigned int g_diag_error = 0;

namespace {

using namespace sm100;

constexpr int CD = 16;               // internal chunk length of the diagonal-gated kernels
constexpr int NP = CD * (CD + 1) / 2;  // pairs j <= i inside a chunk
constexpr int NT = 256;

__device__ __forceinline__ size_t tok_index(int b, int t, int h, int T, int H) {
    return ((size_t)b * T + t) * H + h;
}

// Rows of one 16-token chunk: unit keys, queries, raw log-decays (into Gs, summed afterwards)
// and the per-token coefficients.  One warp per row; rows past the sequence are zero (they then
// contribute nothing and the decays stay flat).
template <int DK, typename Tin>
__device__ __forceinline__ void load_rows(const FwdArgs& a, int b, int h, int t0, int n, float* Ks, float* Qs,
                                          float* Gs, float* bs, float* cs, float* us) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int PER = DK / 32, LDK = DK + 1;
    const Tin* q = static_cast<const Tin*>(a.q);
    const Tin* k = static_cast<const Tin*>(a.k);
    for (int i = warp; i < CD; i += NT / 32) {
        if (i < n) {
            const size_t ti = tok_index(b, t0 + i, h, a.T, a.H);
            float kv[PER];
            float r2 = 0.f;
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                kv[u] = to_f32(k[ti * DK + lane + 32 * u]);
                r2 = fmaf(kv[u], kv[u], r2);
            }
            r2 = warp_sum(r2);
            const float et = a.eta[ti];
            const KaczCoef cf = kacz_coef(et, r2, a.eps);
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                Ks[i * LDK + lane + 32 * u] = kv[u] * cf.inv_r;
                Qs[i * LDK + lane + 32 * u] = to_f32(q[ti * DK + lane + 32 * u]);
                Gs[i * DK + lane + 32 * u] = a.g[ti * DK + lane + 32 * u];
            }
            if (lane == 0) {
                bs[i] = cf.b;
                cs[i] = cf.c;
                // value coefficient of U in the backward: c, except at a key of zero norm, where
                // U's row takes beta v (it meets only khat = 0 there, and row i of dkhat then
                // equals the exact dk = beta Gbar_i v_i)
                if (us) us[i] = r2 == 0.f ? (a.eps < 0.f ? et : (a.eps > 0.f ? et / a.eps : 0.f)) : cf.c;
            }
        } else {
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                Ks[i * LDK + lane + 32 * u] = 0.f;
                Qs[i * LDK + lane + 32 * u] = 0.f;
                Gs[i * DK + lane + 32 * u] = 0.f;
            }
            if (lane == 0) {
                bs[i] = 0.f;
                cs[i] = 0.f;
                if (us) us[i] = 0.f;
            }
        }
    }
}

// Inclusive per-channel prefix sum of the log-decays over the chunk (one thread per channel).
template <int DK>
__device__ __forceinline__ void cumsum_rows(float* Gs) {
    if (threadIdx.x < DK) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < CD; ++i) {
            acc += Gs[i * DK + threadIdx.x];
            Gs[i * DK + threadIdx.x] = acc;
        }
    }
}

// Chunk Gram matrices from the pairwise per-channel decays: A_ij = sum_c khat_i khat_j E_ij
// (j < i) and P_ij = sum_c q_i khat_j E_ij (j <= i).  One warp per pair, lanes over channels.
// When Es is given the factors E_ij[c] are also kept there ([pair][channel]).
template <int DK>
__device__ __forceinline__ void chunk_grams(const float* Ks, const float* Qs, const float* Gs, float* Am, float* Pm,
                                            float* Es) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int PER = DK / 32, LDK = DK + 1, LDC = CD + 1;
    for (int p = warp; p < NP; p += NT / 32) {
        int i = 0;
        while ((i + 1) * (i + 2) / 2 <= p) ++i;
        const int j = p - i * (i + 1) / 2;
        float sa = 0.f, sp = 0.f;
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int c = lane + 32 * u;
            const float e = __expf(Gs[i * DK + c] - Gs[j * DK + c]);
            if (Es) Es[p * DK + c] = e;
            const float kj = Ks[j * LDK + c] * e;
            sa = fmaf(Ks[i * LDK + c], kj, sa);
            sp = fmaf(Qs[i * LDK + c], kj, sp);
        }
        sa = warp_sum(sa);
        sp = warp_sum(sp);
        if (lane == 0) {
            Am[i * LDC + j] = (j < i) ? sa : 0.f;
            Pm[i * LDC + j] = sp;
            if (j < i) {
                Am[j * LDC + i] = 0.f;
                Pm[j * LDC + i] = 0.f;
            } else {
                Am[i * LDC + i] = 0.f;
            }
        }
    }
}

// Per-(head, 16-token chunk) record of the split path (floats; see the split forward below).
template <int DK, int DV>
struct DiagRec {
    static constexpr int kHead = 3 * CD * DK + CD * CD + DK;  // W, QG, KD, P, GC (floats)
    static constexpr int kSlice = CD * 64;                     // one 64-column slice of UP
    static constexpr int kExtra = 2 * CD * CD + CD * DK;       // A, T, G (backward only)
    static constexpr int kFloats = kHead + (DV / 64) * kSlice + kExtra;  // record stride
    static constexpr int W = 0, QG = CD * DK, KD = 2 * CD * DK, P = 3 * CD * DK, GC = 3 * CD * DK + CD * CD,
                         UP = kHead, XA = kHead + (DV / 64) * kSlice, XT = XA + CD * CD, XG = XT + CD * CD;
    static_assert((kHead * 4) % 16 == 0 && (kFloats * 4) % 16 == 0 && (XA * 4) % 16 == 0, "bulk copy alignment");
};

// ------------------------------------------------------------------------------------
// Forward: grid (Dv / NV, H, B); S_chunks (optional) receives the state at the start of every
// 16-token chunk, [B, H, ceil(T/16), Dk, Dv] (the backward's input).
// ------------------------------------------------------------------------------------
template <int DK>
constexpr size_t diag_fwd_smem_bytes() {
    constexpr int NV = 64;
    return sizeof(float) * (3 * CD * (DK + 1) + CD * DK + DK * (NV + 1) + 2 * CD * (NV + 1) + 2 * CD * (CD + 1) +
                            2 * CD);
}

template <int DK, typename Tin, typename TOut>
__global__ void __launch_bounds__(NT, 1) chunk_fwd_diag_kernel(FwdArgs a) {
    constexpr int NV = 64;
    constexpr int LDK = DK + 1, LDV = NV + 1, LDC = CD + 1;
    constexpr int TMS = DK / 16;
    extern __shared__ float sm[];
    float* Ks = sm;               // CD x LDK  unit keys
    float* Qs = Ks + CD * LDK;    // CD x LDK  queries
    float* Ws = Qs + CD * LDK;    // CD x LDK  khat o Gam, later khat o Del
    float* Gs = Ws + CD * LDK;    // CD x DK   log-decay prefix (per channel)
    float* Ss = Gs + CD * DK;     // DK x LDV  state slice
    float* Rs = Ss + DK * LDV;    // CD x LDV  c V -> R -> U
    float* Xs = Rs + CD * LDV;    // CD x LDV  (Khat o Gam) S
    float* Lm = Xs + CD * LDV;    // CD x LDC  L, then P
    float* Pm = Lm + CD * LDC;    // CD x LDC
    float* bs = Pm + CD * LDC;
    float* cs = bs + CD;

    const int v0 = blockIdx.x * NV, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tx = tid & 15, ty = tid >> 4;
    const int T = a.T, H = a.H, Dv = a.Dv;
    const Tin* v = static_cast<const Tin*>(a.v);
    TOut* o = static_cast<TOut*>(a.o);
    const size_t sbase = ((size_t)b * H + h) * DK * Dv;
    const int NC = (T + CD - 1) / CD;

    for (int x = tid; x < DK * NV; x += NT) {
        const int r = x / NV, c = x % NV;
        Ss[r * LDV + c] = a.S0 ? a.S0[sbase + (size_t)r * Dv + v0 + c] : 0.f;
    }

    for (int ci = 0; ci < NC; ++ci) {
        const int t0 = ci * CD;
        const int n = min(CD, T - t0);
        __syncthreads();
        if (a.S_chunks) {
            float* dst = a.S_chunks + (((size_t)b * H + h) * NC + ci) * DK * Dv;
            for (int x = tid; x < DK * NV; x += NT) {
                const int r = x / NV, c = x % NV;
                dst[(size_t)r * Dv + v0 + c] = Ss[r * LDV + c];
            }
        }
        load_rows<DK, Tin>(a, b, h, t0, n, Ks, Qs, Gs, bs, cs, nullptr);
        __syncthreads();
        cumsum_rows<DK>(Gs);
        // c V into Rs
        for (int i = warp; i < CD; i += NT / 32) {
            for (int j = lane; j < NV; j += 32) {
                float val = 0.f;
                if (i < n) val = cs[i] * to_f32(v[tok_index(b, t0 + i, h, T, H) * Dv + v0 + j]);
                Rs[i * LDV + j] = val;
            }
        }
        __syncthreads();
        chunk_grams<DK>(Ks, Qs, Gs, Lm, Pm, nullptr);
        for (int x = tid; x < CD * DK; x += NT) {  // khat o Gam
            const int i = x / DK, c = x % DK;
            Ws[i * LDK + c] = Ks[i * LDK + c] * __expf(Gs[i * DK + c]);
        }
        __syncthreads();
        // X = (Khat o Gam) S: one row per ty, four columns per thread
        {
            float ax[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int d = 0; d < DK; ++d) {
                const float w = Ws[ty * LDK + d];
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) ax[nn] = fmaf(w, Ss[d * LDV + tx + 16 * nn], ax[nn]);
            }
#pragma unroll
            for (int nn = 0; nn < 4; ++nn) Xs[ty * LDV + tx + 16 * nn] = ax[nn];
        }
        __syncthreads();
        // R = c V - Diag(b) X; L = Diag(b) A
        for (int x = tid; x < CD * NV; x += NT) {
            const int i = x / NV, j = x % NV;
            Rs[i * LDV + j] -= bs[i] * Xs[i * LDV + j];
        }
        if (tid < CD * CD) {
            const int i = tid / CD, j = tid % CD;
            Lm[i * LDC + j] *= bs[i];
        }
        __syncthreads();
        // Forward substitution (I + L) U = R, row by row (Appendix B.2)
        {
            const int col = tid >> 2, part = tid & 3;
            for (int i = 1; i < n; ++i) {
                if (col < NV) {
                    float s = 0.f;
                    for (int j = part; j < i; j += 4) s = fmaf(Lm[i * LDC + j], Rs[j * LDV + col], s);
                    s += __shfl_xor_sync(0xffffffffu, s, 1);
                    s += __shfl_xor_sync(0xffffffffu, s, 2);
                    if (part == 0) Rs[i * LDV + col] -= s;
                }
                __syncthreads();
            }
        }
        // O = (Q o Gam) S + P U
        if (o != nullptr) {
            float ao[4] = {0.f, 0.f, 0.f, 0.f};
            const int i = ty;
#pragma unroll 4
            for (int d = 0; d < DK; ++d) {
                const float w = Qs[i * LDK + d] * __expf(Gs[i * DK + d]);
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) ao[nn] = fmaf(w, Ss[d * LDV + tx + 16 * nn], ao[nn]);
            }
#pragma unroll
            for (int t = 0; t < CD; ++t) {
                const float p = Pm[i * LDC + t];
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) ao[nn] = fmaf(p, Rs[t * LDV + tx + 16 * nn], ao[nn]);
            }
            if (i < n) {
                TOut* orow = o + tok_index(b, t0 + i, h, T, H) * Dv + v0;
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) orow[tx + 16 * nn] = from_f32<TOut>(ao[nn]);
            }
        }
        // khat o Del, Del_j = exp(G_last - G_j)
        for (int x = tid; x < CD * DK; x += NT) {
            const int i = x / DK, c = x % DK;
            Ws[i * LDK + c] = Ks[i * LDK + c] * __expf(Gs[(n - 1) * DK + c] - Gs[i * DK + c]);
        }
        __syncthreads();
        // S' = Diag(Gam_last) S + (Khat o Del)^T U
        {
            float as[TMS][4];
#pragma unroll
            for (int m = 0; m < TMS; ++m)
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) as[m][nn] = 0.f;
#pragma unroll
            for (int t = 0; t < CD; ++t) {
                float uu[4];
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) uu[nn] = Rs[t * LDV + tx + 16 * nn];
#pragma unroll
                for (int m = 0; m < TMS; ++m) {
                    const float w = Ws[t * LDK + ty + 16 * m];
#pragma unroll
                    for (int nn = 0; nn < 4; ++nn) as[m][nn] = fmaf(w, uu[nn], as[m][nn]);
                }
            }
#pragma unroll
            for (int m = 0; m < TMS; ++m) {
                const int r = ty + 16 * m;
                const float gl_r = __expf(Gs[(n - 1) * DK + r]);
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) {
                    float* sp = &Ss[r * LDV + tx + 16 * nn];
                    *sp = fmaf(gl_r, *sp, as[m][nn]);
                }
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

// ------------------------------------------------------------------------------------
// Backward.  Per chunk (newest first) with incoming state S and lambda = dS' (gradient of the
// outgoing state), Gam_i = exp(G_i), Del_j = exp(G_last - G_j) (vectors over channels), and
// the forward preparation's record of the chunk (W, QG = Q o Gam, KD = Khat o Del, P, GC, UP,
// A, T, G):
//   U   = UP - W S + Diag(u - c) V     (u = c except at a zero-norm key, where u = beta: see below)
//   dU  = P^T dO + KD lambda,   dR = T^T dU
//   dS  = Diag(GC) lambda + QG^T dO - W^T dU                                     (carried on)
//   dv  = Diag(c) dR,  dc_i = dR_i . v_i
//   Y   = dO U^T (lower),  D = -dR U^T (strictly lower)
//   Z1 = dO S^T, Z2 = dR S^T, Z3 = U lambda^T                     (rows: tokens, columns: channels)
//   F1_i = sum_{j<=i} Y_ij khat_j o E_ij     F2_j = sum_{i>=j} Y_ij q_i o E_ij
//   F3_i = sum_{j<i}  D_ij khat_j o E_ij     F4_j = sum_{i>j}  D_ij b_i khat_i o E_ij
//   dq_i    = Gam_i o Z1_i + F1_i
//   dkhat_i = -b_i Gam_i o Z2_i + Del_i o Z3_i + F2_i + b_i F3_i + F4_i
//   db_i    = sum_{j<i} D_ij A_ij - (khat_i o Gam_i) . Z2_i
//   dG_i    = Gam_i o q_i o Z1_i + q_i o F1_i - b_i Gam_i o khat_i o Z2_i - khat_i o F2_i
//             + b_i khat_i o F3_i - khat_i o F4_i - Del_i o khat_i o Z3_i
//   dG_last += sum_j Del_j o khat_j o Z3_j + GC o rowsum(lambda o S)
// (W^T dU = (T Diag(b)(Khat o Gam))^T dU = (Diag(b)(Khat o Gam))^T dR.)  At a key of zero norm
// U's row takes u = beta v: that row only ever meets khat = 0, except in row i of dkhat, which
// then is the exact dk = beta Gbar_i v_i.  One CTA per (head, 64 value columns); the columns'
// partial sums of dq, dkhat, dG, db and dc go out by vector reductions into fp32 accumulators.
// ------------------------------------------------------------------------------------
constexpr int BLD = 68;  // row stride of the [rows][64] fp32 tiles (16-byte rows, 2-way banks)
constexpr float kFactorLimit = 80.f;  // |G| below this: exp(+-G) and their products stay finite in fp32

// Shared memory of the backward (floats, then the raw rows of the next chunk, then barriers).
template <int DK, int DV, typename Tin>
constexpr size_t diag_bwd_smem_bytes() {
    using R = DiagRec<DK, DV>;
    return 128 + sizeof(float) * ((size_t)2 * DK * BLD + 6 * CD * DK + R::kHead + R::kExtra + CD * 64 +
                                  2 * CD * (DK + 1) + 5 * CD * BLD + 2 * CD * (CD + 1) + DK + 5 * CD) +
           sizeof(Tin) * (size_t)CD * (2 * DK + 128) + 16 + 3 * 8;
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// Per chunk the pairwise factors E_ij = exp(G_i - G_j) enter the F terms only through products
// with per-token rows, so while every |G| of the chunk is below kFactorLimit they are taken as
// exp(G_i) exp(-G_j):
//   F1_i = Gam_i o sum_{j<=i} Y_ij (khat_j o Gam_j^-1)      F3_i likewise with D
//   F2_j = Gam_j^-1 o sum_{i>=j} Y_ij (q_i o Gam_i)         F4_j = Gam_j^-1 o sum_{i>j} D_ij b_i (khat_i o Gam_i)
// (q o Gam is the record's QG).  A chunk with a wider range forms each E_ij on the fly instead.
// The rows of the next chunk (k, q, and this CTA's v and dO columns) come in by bulk copies
// while the current one is worked on.
template <int DK, int DV, typename Tin, typename TOut>
__global__ void __launch_bounds__(NT, 1) diag_bwd_kernel(BwdArgs a, FwdArgs f, const float* __restrict__ recs) {
    using R = DiagRec<DK, DV>;
    constexpr int LDK = DK + 1, LDC = CD + 1;
    constexpr int EPT = CD * DK / NT;  // (token, channel) elements per thread: tx + 16 u
    extern __shared__ uint8_t smem_raw[];
    float* sm = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    float* Ss = sm;                      // DK x BLD  incoming state slice
    float* Ls = Ss + DK * BLD;           // DK x BLD  lambda slice
    float* Rq = Ls + DK * BLD;           // CD x DK   results: dq, dkhat, dG, last-token terms
    float* Rk = Rq + CD * DK;
    float* Rg = Rk + CD * DK;
    float* Rxs = Rg + CD * DK;
    float* KiG = Rxs + CD * DK;          // CD x DK   khat o Gam^-1
    float* KG = KiG + CD * DK;           // CD x DK   khat o Gam
    float* Rh = KG + CD * DK;            // record head: W, QG, KD, P, GC
    float* Rx = Rh + R::kHead;           // record extras: A, T, G
    float* UPs = Rx + R::kExtra;         // CD x 64   UP slice
    float* Kh = UPs + CD * 64;           // CD x LDK  unit keys
    float* Qs = Kh + CD * LDK;           // CD x LDK
    float* Us = Qs + CD * LDK;           // CD x BLD
    float* dUs = Us + CD * BLD;          // CD x BLD
    float* dRs = dUs + CD * BLD;         // CD x BLD
    float* dOs = dRs + CD * BLD;         // CD x BLD
    float* Vs = dOs + CD * BLD;          // CD x BLD
    float* Ym = Vs + CD * BLD;           // CD x LDC
    float* Dm = Ym + CD * LDC;           // CD x LDC
    float* lsS = Dm + CD * LDC;          // DK
    float* bs = lsS + DK;
    float* cs = bs + CD;
    float* us = cs + CD;
    float* dbs = us + CD;
    float* etaS = dbs + CD;
    Tin* Kraw = reinterpret_cast<Tin*>((reinterpret_cast<uintptr_t>(etaS + CD) + 15) & ~uintptr_t(15));
    Tin* Qraw = Kraw + CD * DK;          // raw rows of the next chunk: k, q [CD][DK]
    Tin* Vraw = Qraw + CD * DK;          // v, dO columns v0 .. v0 + 63 [CD][64]
    Tin* Oraw = Vraw + CD * 64;
    uint64_t* bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(Oraw + CD * 64) + 15) & ~uintptr_t(15));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sl = blockIdx.x, v0 = sl * 64, h = blockIdx.y, b = blockIdx.z;
    const int T = a.T, H = a.H;
    const int NC = (T + CD - 1) / CD;
    const size_t head = (size_t)b * H + h;
    const size_t sbase = head * DK * DV;
    const float* hrec = recs + head * NC * R::kFloats;
    const Tin* kin = static_cast<const Tin*>(f.k);
    const Tin* qin = static_cast<const Tin*>(f.q);
    const Tin* v = static_cast<const Tin*>(a.v);
    const Tin* dO = static_cast<const Tin*>(a.dO);
    TOut* dv = static_cast<TOut*>(a.dv);
    const uint32_t bar_r = smem_u32(&bars[0]), bar_s = smem_u32(&bars[1]), bar_x = smem_u32(&bars[2]);

    // the chunk's record parts (head, its UP slice, extras): one thread
    auto request_rec = [&](int c) {
        const float* r = hrec + (size_t)c * R::kFloats;
        mbar_expect_tx(bar_r, (R::kHead + CD * 64 + R::kExtra) * 4);
        bulk_load(smem_u32(Rh), r, R::kHead * 4, bar_r);
        bulk_load(smem_u32(UPs), r + R::UP + sl * R::kSlice, CD * 64 * 4, bar_r);
        bulk_load(smem_u32(Rx), r + R::XA, R::kExtra * 4, bar_r);
    };
    // the incoming state's slice rows of chunk c: warp 0, rows split over the lanes
    auto request_state = [&](int c) {
        const float* src = a.S_chunks + (head * NC + c) * DK * DV + v0;
        if (lane == 0) mbar_expect_tx(bar_s, DK * 64 * 4);
        __syncwarp();
        for (int r = lane; r < DK; r += 32) bulk_load(smem_u32(Ss + r * BLD), src + (size_t)r * DV, 256, bar_s);
    };
    // raw rows of chunk c (k, q, v and dO columns of this CTA): warp 0, one token per lane
    auto request_raw = [&](int c) {
        const int tc = c * CD, nc = min(CD, T - tc);
        if (lane == 0) mbar_expect_tx(bar_x, (uint32_t)(nc * (2 * DK + 128) * sizeof(Tin)));
        __syncwarp();
        if (lane < nc) {
            const size_t ti = tok_index(b, tc + lane, h, T, H);
            bulk_load(smem_u32(Kraw + lane * DK), kin + ti * DK, DK * sizeof(Tin), bar_x);
            bulk_load(smem_u32(Qraw + lane * DK), qin + ti * DK, DK * sizeof(Tin), bar_x);
            bulk_load(smem_u32(Vraw + lane * 64), v + ti * DV + v0, 64 * sizeof(Tin), bar_x);
            bulk_load(smem_u32(Oraw + lane * 64), dO + ti * DV + v0, 64 * sizeof(Tin), bar_x);
        }
    };
    if (tid == 0) {
        mbar_init(bar_r, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_x, 1);
        fence_mbar_init();
        if (NC > 0) request_rec(NC - 1);
    }
    if (tid < CD) {  // the newest chunk's eta (later chunks' come a chunk ahead)
        const int t = (NC - 1) * CD + tid;
        etaS[tid] = t < T ? f.eta[tok_index(b, t, h, T, H)] : 0.f;
    }
    for (int x = tid; x < DK * 64; x += NT) {
        const int r = x >> 6, c = x & 63;
        Ls[r * BLD + c] = a.dS_T ? a.dS_T[sbase + (size_t)r * DV + v0 + c] : 0.f;
    }
    __syncthreads();  // barriers initialised
    if (warp == 0 && NC > 0) {
        request_state(NC - 1);
        request_raw(NC - 1);
    }

    const int i = tid >> 4, tx = tid & 15, cx = 4 * tx;  // token row and this thread's columns
    bool ok = true;
    int ci_stop = 0, stop_kind = 0;  // where a bounded wait gave up (for the drain below)
    for (int ci = NC - 1; ci >= 0; --ci) {
        const int t0 = ci * CD, n = min(CD, T - t0);
        const int ph = (NC - 1 - ci) & 1;
        float eta_next = 0.f;  // the next (older, always full) chunk's eta, stored once etaS is read
        if (tid < CD && ci > 0) eta_next = f.eta[tok_index(b, t0 - CD + tid, h, T, H)];
        __syncthreads();
        const bool gotx = mbar_wait_bounded(bar_x, ph, 2000000000ull);
        if (__syncthreads_or(!gotx)) {
            ok = false;
            ci_stop = ci;
            stop_kind = 0;
            break;
        }
        // ---- rows of the chunk: unit keys, queries, coefficients (u: the U coefficient); v, dO
        for (int r = warp; r < CD; r += NT / 32) {
            constexpr int PER = DK / 32;
            if (r < n) {
                float kv[PER];
                float r2 = 0.f;
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    kv[u] = to_f32(Kraw[r * DK + lane + 32 * u]);
                    r2 = fmaf(kv[u], kv[u], r2);
                }
                r2 = warp_sum(r2);
                const float et = etaS[r];
                const KaczCoef cf = kacz_coef(et, r2, f.eps);
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    Kh[r * LDK + lane + 32 * u] = kv[u] * cf.inv_r;
                    Qs[r * LDK + lane + 32 * u] = to_f32(Qraw[r * DK + lane + 32 * u]);
                }
                if (lane == 0) {
                    bs[r] = cf.b;
                    cs[r] = cf.c;
                    // U's value coefficient in the backward: c, except at a key of zero norm, where
                    // U's row takes beta v (that row meets only khat = 0, except in row r of dkhat,
                    // which then equals the exact dk = beta Gbar_r v_r)
                    us[r] = r2 == 0.f ? (f.eps < 0.f ? et : (f.eps > 0.f ? et / f.eps : 0.f)) : cf.c;
                }
            } else {
#pragma unroll
                for (int u = 0; u < PER; ++u) {
                    Kh[r * LDK + lane + 32 * u] = 0.f;
                    Qs[r * LDK + lane + 32 * u] = 0.f;
                }
                if (lane == 0) bs[r] = cs[r] = us[r] = 0.f;
            }
        }
        for (int x = tid; x < CD * 16; x += NT) {
            const int r = x >> 4, c4 = 4 * (x & 15);
            float vv[4] = {0.f, 0.f, 0.f, 0.f}, oo[4] = {0.f, 0.f, 0.f, 0.f};
            if (r < n) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    vv[e] = to_f32(Vraw[r * 64 + c4 + e]);
                    oo[e] = to_f32(Oraw[r * 64 + c4 + e]);
                }
            }
            *reinterpret_cast<float4*>(Vs + r * BLD + c4) = make_float4(vv[0], vv[1], vv[2], vv[3]);
            *reinterpret_cast<float4*>(dOs + r * BLD + c4) = make_float4(oo[0], oo[1], oo[2], oo[3]);
        }
        if (tid < CD) dbs[tid] = 0.f;
        __syncthreads();  // the raw rows and etaS are read: the next chunk's may come in
        if (warp == 0 && ci > 0) request_raw(ci - 1);
        if (tid < CD) etaS[tid] = eta_next;
        const bool got = mbar_wait_bounded(bar_r, ph, 2000000000ull) && mbar_wait_bounded(bar_s, ph, 2000000000ull);
        if (__syncthreads_or(!got)) {
            ok = false;
            ci_stop = ci;
            stop_kind = 1;
            break;
        }
        const float* Gs = Rx + (R::XG - R::XA);
        const float* Am = Rx;
        const float* Tm = Rx + CD * CD;
        const float* QGr = Rh + R::QG;
        // ---- per-token decay factors of the keys, and whether the chunk's range allows them
        bool wide = false;
        for (int x = tid; x < CD * DK; x += NT) {
            const int t = x / DK, d = x % DK;
            const float G = Gs[x];
            wide |= !(fabsf(G) < kFactorLimit);
            const float kh = Kh[t * LDK + d];
            KiG[x] = kh * __expf(-G);
            KG[x] = kh * __expf(G);
        }
        // ---- U = UP - W S + (u - c) v  and  dU = P^T dO + KD lambda (row i, columns cx .. cx + 3)
        {
            float4 u = *reinterpret_cast<const float4*>(UPs + i * 64 + cx);
            float4 du = make_float4(0.f, 0.f, 0.f, 0.f);
            const float* wr = Rh + R::W + i * DK;
            const float* kr = Rh + R::KD + i * DK;
#pragma unroll 4
            for (int d = 0; d < DK; ++d) {
                const float w = wr[d], kd = kr[d];
                const float4 s4 = *reinterpret_cast<const float4*>(Ss + d * BLD + cx);
                const float4 l4 = *reinterpret_cast<const float4*>(Ls + d * BLD + cx);
                u.x = fmaf(-w, s4.x, u.x); u.y = fmaf(-w, s4.y, u.y); u.z = fmaf(-w, s4.z, u.z); u.w = fmaf(-w, s4.w, u.w);
                du.x = fmaf(kd, l4.x, du.x); du.y = fmaf(kd, l4.y, du.y); du.z = fmaf(kd, l4.z, du.z); du.w = fmaf(kd, l4.w, du.w);
            }
            const float* pc = Rh + R::P + i;  // column i of P
#pragma unroll
            for (int t = 0; t < CD; ++t) {
                const float pt = pc[t * CD];
                const float4 o4 = *reinterpret_cast<const float4*>(dOs + t * BLD + cx);
                du.x = fmaf(pt, o4.x, du.x); du.y = fmaf(pt, o4.y, du.y); du.z = fmaf(pt, o4.z, du.z); du.w = fmaf(pt, o4.w, du.w);
            }
            const float zc = us[i] - cs[i];
            if (zc != 0.f) {
                const float4 v4 = *reinterpret_cast<const float4*>(Vs + i * BLD + cx);
                u.x = fmaf(zc, v4.x, u.x); u.y = fmaf(zc, v4.y, u.y); u.z = fmaf(zc, v4.z, u.z); u.w = fmaf(zc, v4.w, u.w);
            }
            *reinterpret_cast<float4*>(Us + i * BLD + cx) = u;
            *reinterpret_cast<float4*>(dUs + i * BLD + cx) = du;
        }
        wide = __syncthreads_or(wide);
        // ---- dR = T^T dU (row j = i here); lambda o S row sums
        {
            float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int t = i; t < CD; ++t) {
                const float tt = Tm[t * CD + i];
                const float4 d4 = *reinterpret_cast<const float4*>(dUs + t * BLD + cx);
                r4.x = fmaf(tt, d4.x, r4.x); r4.y = fmaf(tt, d4.y, r4.y); r4.z = fmaf(tt, d4.z, r4.z); r4.w = fmaf(tt, d4.w, r4.w);
            }
            *reinterpret_cast<float4*>(dRs + i * BLD + cx) = r4;
        }
        // rows of lambda o S summed: sixteen lanes per row, each a 4-column group (whole 256-byte
        // rows per half-warp, no bank conflicts), then a 16-lane shuffle sum
        for (int d = tid >> 4; d < DK; d += NT / 16) {
            const float4 l4 = *reinterpret_cast<const float4*>(Ls + d * BLD + cx);
            const float4 s4 = *reinterpret_cast<const float4*>(Ss + d * BLD + cx);
            float p = l4.x * s4.x + l4.y * s4.y + l4.z * s4.z + l4.w * s4.w;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            if (tx == 0) lsS[d] = p;
        }
        __syncthreads();
        // ---- dv, dc; Y, D; the D o A part of db
        {
            const float4 r4 = *reinterpret_cast<const float4*>(dRs + i * BLD + cx);
            const float4 v4 = *reinterpret_cast<const float4*>(Vs + i * BLD + cx);
            float dcp = r4.x * v4.x + r4.y * v4.y + r4.z * v4.z + r4.w * v4.w;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) dcp += __shfl_xor_sync(0xffffffffu, dcp, o);
            if (i < n) {
                const size_t ti = tok_index(b, t0 + i, h, T, H);
                const float ci_ = cs[i];
                TOut* dvr = dv + ti * DV + v0 + cx;
                dvr[0] = from_f32<TOut>(ci_ * r4.x);
                dvr[1] = from_f32<TOut>(ci_ * r4.y);
                dvr[2] = from_f32<TOut>(ci_ * r4.z);
                dvr[3] = from_f32<TOut>(ci_ * r4.w);
                if (tx == 0) atomicAdd(&a.acc_dc[ti], dcp);
            }
            const int j = tx;
            float y = 0.f, dd = 0.f;
#pragma unroll 4
            for (int c = 0; c < 64; c += 4) {
                const float4 uj = *reinterpret_cast<const float4*>(Us + j * BLD + c);
                const float4 oi = *reinterpret_cast<const float4*>(dOs + i * BLD + c);
                const float4 ri = *reinterpret_cast<const float4*>(dRs + i * BLD + c);
                y += oi.x * uj.x + oi.y * uj.y + oi.z * uj.z + oi.w * uj.w;
                dd += ri.x * uj.x + ri.y * uj.y + ri.z * uj.z + ri.w * uj.w;
            }
            const float Y = (j <= i) ? y : 0.f, D = (j < i) ? -dd : 0.f;
            Ym[i * LDC + j] = Y;
            Dm[i * LDC + j] = D;
            float da = D * Am[i * CD + j];
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) da += __shfl_xor_sync(0xffffffffu, da, o);
            if (tx == 0) dbs[i] = da;
        }
        // ---- Z1 = dO S^T, Z2 = dR S^T, Z3 = U lambda^T: warp w takes token rows 2w and 2w + 1,
        //      lane l channels l + 32 v (a warp reads whole rows: no bank conflicts, and the row
        //      operands are broadcast)
        constexpr int NVC = DK / 32;
        const int rw = 2 * warp;
        float zq[2][NVC], zr[2][NVC], zl[2][NVC];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
            for (int v = 0; v < NVC; ++v) zq[h2][v] = zr[h2][v] = zl[h2][v] = 0.f;
#pragma unroll 2
        for (int c = 0; c < 64; c += 4) {
            float4 o4[2], r4[2], u4[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                o4[h2] = *reinterpret_cast<const float4*>(dOs + (rw + h2) * BLD + c);
                r4[h2] = *reinterpret_cast<const float4*>(dRs + (rw + h2) * BLD + c);
                u4[h2] = *reinterpret_cast<const float4*>(Us + (rw + h2) * BLD + c);
            }
#pragma unroll
            for (int v = 0; v < NVC; ++v) {
                const int d = lane + 32 * v;
                const float4 s4 = *reinterpret_cast<const float4*>(Ss + d * BLD + c);
                const float4 l4 = *reinterpret_cast<const float4*>(Ls + d * BLD + c);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    zq[h2][v] += o4[h2].x * s4.x + o4[h2].y * s4.y + o4[h2].z * s4.z + o4[h2].w * s4.w;
                    zr[h2][v] += r4[h2].x * s4.x + r4[h2].y * s4.y + r4[h2].z * s4.z + r4[h2].w * s4.w;
                    zl[h2][v] += u4[h2].x * l4.x + u4[h2].y * l4.y + u4[h2].z * l4.z + u4[h2].w * l4.w;
                }
            }
        }
        __syncthreads();  // Ym, Dm written; S read: the previous chunk's state may come in
        if (warp == 0 && ci > 0) request_state(ci - 1);
        // ---- F terms and the per-(token, channel) gradients, row by row of the warp's two
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int ii = rw + h2;
            float f1[NVC], f2[NVC], f3[NVC], f4[NVC];
#pragma unroll
            for (int v = 0; v < NVC; ++v) f1[v] = f2[v] = f3[v] = f4[v] = 0.f;
            if (!wide) {
                for (int j = 0; j <= ii; ++j) {
                    const float y = Ym[ii * LDC + j], dd = Dm[ii * LDC + j];
#pragma unroll
                    for (int v = 0; v < NVC; ++v) {
                        const float kig = KiG[j * DK + lane + 32 * v];
                        f1[v] = fmaf(y, kig, f1[v]);
                        f3[v] = fmaf(dd, kig, f3[v]);
                    }
                }
                for (int r = ii; r < n; ++r) {
                    const float y = Ym[r * LDC + ii], dd = Dm[r * LDC + ii] * bs[r];
#pragma unroll
                    for (int v = 0; v < NVC; ++v) {
                        const int d = lane + 32 * v;
                        f2[v] = fmaf(y, QGr[r * DK + d], f2[v]);
                        f4[v] = fmaf(dd, KG[r * DK + d], f4[v]);
                    }
                }
#pragma unroll
                for (int v = 0; v < NVC; ++v) {
                    const float G = Gs[ii * DK + lane + 32 * v];
                    const float gp = __expf(G), gm = __expf(-G);
                    f1[v] *= gp;
                    f3[v] *= gp;
                    f2[v] *= gm;
                    f4[v] *= gm;
                }
            } else {
                for (int j = 0; j <= ii; ++j) {
                    const float y = Ym[ii * LDC + j], dd = Dm[ii * LDC + j];
#pragma unroll
                    for (int v = 0; v < NVC; ++v) {
                        const int d = lane + 32 * v;
                        const float ke = Kh[j * LDK + d] * __expf(Gs[ii * DK + d] - Gs[j * DK + d]);
                        f1[v] = fmaf(y, ke, f1[v]);
                        f3[v] = fmaf(dd, ke, f3[v]);
                    }
                }
                for (int r = ii; r < n; ++r) {
                    const float y = Ym[r * LDC + ii], dd = Dm[r * LDC + ii] * bs[r];
#pragma unroll
                    for (int v = 0; v < NVC; ++v) {
                        const int d = lane + 32 * v;
                        const float e = __expf(Gs[r * DK + d] - Gs[ii * DK + d]);
                        f2[v] = fmaf(y, Qs[r * LDK + d] * e, f2[v]);
                        f4[v] = fmaf(dd, Kh[r * LDK + d] * e, f4[v]);
                    }
                }
            }
            const float bi = bs[ii];
            float kgz = 0.f;
#pragma unroll
            for (int v = 0; v < NVC; ++v) {
                const int d = lane + 32 * v;
                const float G = Gs[ii * DK + d], Gl = Gs[(n - 1) * DK + d];
                const float gam = __expf(G), del = __expf(Gl - G);
                const float qd = Qs[ii * LDK + d], kd = Kh[ii * LDK + d];
                Rq[ii * DK + d] = fmaf(gam, zq[h2][v], f1[v]);
                Rk[ii * DK + d] = -bi * gam * zr[h2][v] + del * zl[h2][v] + f2[v] + bi * f3[v] + f4[v];
                Rg[ii * DK + d] = gam * qd * zq[h2][v] + qd * f1[v] - bi * gam * kd * zr[h2][v] - kd * f2[v] +
                                  bi * kd * f3[v] - kd * f4[v] - del * kd * zl[h2][v];
                Rxs[ii * DK + d] = (ii < n) ? del * kd * zl[h2][v] : 0.f;
                kgz = fmaf(kd * gam, zr[h2][v], kgz);
            }
            kgz = warp_sum(kgz);
            if (lane == 0) dbs[ii] -= kgz;
        }
        // ---- new lambda = Diag(GC) lambda + QG^T dO - W^T dU (rows i + 16 m, columns cx .. cx + 3);
        //      every other read of lambda was before the last barrier
        {
            float4 acc[DK / 16];
#pragma unroll
            for (int m = 0; m < DK / 16; ++m) {
                const int r = i + 16 * m;
                const float gc = Rh[R::GC + r];
                const float4 l4 = *reinterpret_cast<const float4*>(Ls + r * BLD + cx);
                acc[m] = make_float4(gc * l4.x, gc * l4.y, gc * l4.z, gc * l4.w);
            }
#pragma unroll
            for (int t = 0; t < CD; ++t) {
                const float4 o4 = *reinterpret_cast<const float4*>(dOs + t * BLD + cx);
                const float4 d4 = *reinterpret_cast<const float4*>(dUs + t * BLD + cx);
                const float* qg = Rh + R::QG + t * DK + i;
                const float* wr = Rh + R::W + t * DK + i;
#pragma unroll
                for (int m = 0; m < DK / 16; ++m) {
                    const float wq = qg[16 * m], ww = wr[16 * m];
                    acc[m].x = fmaf(wq, o4.x, fmaf(-ww, d4.x, acc[m].x));
                    acc[m].y = fmaf(wq, o4.y, fmaf(-ww, d4.y, acc[m].y));
                    acc[m].z = fmaf(wq, o4.z, fmaf(-ww, d4.z, acc[m].z));
                    acc[m].w = fmaf(wq, o4.w, fmaf(-ww, d4.w, acc[m].w));
                }
            }
#pragma unroll
            for (int m = 0; m < DK / 16; ++m) *reinterpret_cast<float4*>(Ls + (i + 16 * m) * BLD + cx) = acc[m];
        }
        __syncthreads();
        if (tid < DK) {  // dG of the last token: sum_j Del_j o khat_j o Z3_j + GC o rowsum(lambda o S)
            float e = Rh[R::GC + tid] * lsS[tid];
            for (int r = 0; r < n; ++r) e += Rxs[r * DK + tid];
            Rg[(n - 1) * DK + tid] += e;
        }
        __syncthreads();
        // ---- out: dq, dkhat, dG of this chunk's tokens (eight consecutive channels a thread)
        for (int x = tid; x < CD * DK / 8; x += NT) {
            const int r = x / (DK / 8), c8 = 8 * (x % (DK / 8));
            if (r < n) {
                const size_t o = tok_index(b, t0 + r, h, T, H) * DK + c8;
                const float* pq = Rq + r * DK + c8;
                const float* pk = Rk + r * DK + c8;
                const float* pg = Rg + r * DK + c8;
                red_add_v4(a.acc_dq + o, pq[0], pq[1], pq[2], pq[3]);
                red_add_v4(a.acc_dq + o + 4, pq[4], pq[5], pq[6], pq[7]);
                red_add_v4(a.acc_dkh + o, pk[0], pk[1], pk[2], pk[3]);
                red_add_v4(a.acc_dkh + o + 4, pk[4], pk[5], pk[6], pk[7]);
                red_add_v4(a.acc_dG + o, pg[0], pg[1], pg[2], pg[3]);
                red_add_v4(a.acc_dG + o + 4, pg[4], pg[5], pg[6], pg[7]);
            }
        }
        if (tid < n) atomicAdd(&a.acc_db[tok_index(b, t0 + tid, h, T, H)], dbs[tid]);
        if (tid == 0 && ci > 0) request_rec(ci - 1);  // every read of the record is done
    }
    if (!ok && tid == 0) {
        atomicOr(&g_diag_error, 2u);
        // let copies still in flight land before the block exits: the stopped chunk's record,
        // state and rows, and the older chunk's rows when they were already requested (a wait
        // on a phase that has completed returns at once)
        const int ph = (NC - 1 - ci_stop) & 1;
        (void)mbar_wait_bounded(bar_x, ph, 2000000000ull);
        (void)mbar_wait_bounded(bar_r, ph, 2000000000ull);
        (void)mbar_wait_bounded(bar_s, ph, 2000000000ull);
        if (stop_kind == 1 && ci_stop > 0) (void)mbar_wait_bounded(bar_x, ph ^ 1, 2000000000ull);
    }
    __syncthreads();
    if (ok) {
        for (int x = tid; x < DK * 64; x += NT) {
            const int r = x >> 6, c = x & 63;
            a.dS0[sbase + (size_t)r * DV + v0 + c] = Ls[r * BLD + c];
        }
    }
}

// dq to the output type; dk and deta from the unit-key gradients (as for scalar gating):
//   deta = db r^2/den + dc r/den,  dr = db eta 2 r eps/den^2 + dc eta (eps - r^2)/den^2
//   dk   = (dkhat - khat (khat . dkhat)) / r + khat dr;  at a key of zero norm dkhat already is dk
template <int DK, typename Tin, typename TOut>
__global__ void __launch_bounds__(256) diag_finalize_kernel(BwdArgs a, size_t ntok) {
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
    const bool direct = a.eps < 0.f;
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

// dg_r[c] = sum_{i >= r} dG_i[c] inside each 16-token chunk (one thread per chunk and channel).
template <int DK>
__global__ void diag_dg_kernel(BwdArgs a) {
    const int NC = (a.T + CD - 1) / CD;
    const size_t id = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t total = (size_t)a.B * a.H * NC * DK;
    if (id >= total) return;
    const int c = (int)(id % DK);
    const size_t ch = id / DK;
    const int h = (int)(ch % a.H);
    const int ci = (int)((ch / a.H) % NC);
    const int b = (int)(ch / ((size_t)a.H * NC));
    const int t0 = ci * CD;
    const int n = min(CD, a.T - t0);
    float acc = 0.f;
    for (int i = n - 1; i >= 0; --i) {
        const size_t ti = tok_index(b, t0 + i, h, a.T, a.H) * DK + c;
        acc += a.acc_dG[ti];
        a.dg[ti] = acc;
    }
}

// ------------------------------------------------------------------------------------
// Split forward.  `diag_prep_kernel` (one CTA per 16-token chunk and head, all at once) forms
// everything that does not depend on the incoming state and stores it as an fp32 record:
//   W  = T Diag(b) (Khat o Gam)   [16][DK]     T = (I + L)^{-1}
//   QG = Q o Gam                  [16][DK]
//   KD = Khat o Del               [16][DK]
//   P                             [16][16]
//   GC = Gam_last                 [DK]
//   UP = T Diag(c) V              [DV/64][16][64]   (in 64-column slices)
// and, for the backward, A [16][16] (Gram without b), T [16][16] and G [16][DK].
// `diag_state_kernel` then walks each head's chunks in order on a 64-column slice of the state:
//   U = UP - W S,   O = QG S + P U,   S' = Diag(GC) S + KD^T U,
// with the records double-buffered in shared memory by bulk copies.
// ------------------------------------------------------------------------------------

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(NT) diag_prep_kernel(FwdArgs a, float* __restrict__ recs) {
    using R = DiagRec<DK, DV>;
    constexpr int LDK = DK + 1, LDC = CD + 1;
    constexpr int NR = DK + DV + CD;  // right-hand sides: Diag(b)(Khat o Gam) | Diag(c) V | I
    constexpr int LDR = NR + 1;
    constexpr int NQ = 4;             // channel quarters of the Gram sums
    extern __shared__ float sm[];
    float* Ks = sm;               // CD x LDK  unit keys
    float* Qs = Ks + CD * LDK;    // CD x LDK  queries
    float* Gs = Qs + CD * LDK;    // CD x DK   log-decay prefix
    float* Rs = Gs + CD * DK;     // CD x LDR  right-hand sides, solved in place: W | UP | T
    float* Ap = Rs + CD * LDR;    // NQ x NP   partial Gram sums (A), then
    float* Pp = Ap + NQ * NP;     // NQ x NP   (P)
    float* Am = Pp + NQ * NP;     // CD x LDC  A (strictly lower)
    float* bs = Am + CD * LDC;
    float* cs = bs + CD;

    const int tid = threadIdx.x;
    const int ci = blockIdx.x, head = blockIdx.y;
    const int b = head / a.H, h = head % a.H;
    const int NC = (a.T + CD - 1) / CD;
    const int t0 = ci * CD, n = min(CD, a.T - t0);
    float* rec = recs + ((size_t)head * NC + ci) * R::kFloats;
    const Tin* v = static_cast<const Tin*>(a.v);

    load_rows<DK, Tin>(a, b, h, t0, n, Ks, Qs, Gs, bs, cs, nullptr);
    __syncthreads();
    cumsum_rows<DK>(Gs);
    for (int x = tid; x < CD * DV; x += NT) {  // Diag(c) V
        const int i = x / DV, j = x % DV;
        Rs[i * LDR + DK + j] = i < n ? cs[i] * to_f32(v[tok_index(b, t0 + i, h, a.T, a.H) * DV + j]) : 0.f;
    }
    for (int x = tid; x < CD * CD; x += NT) Rs[(x / CD) * LDR + DK + DV + x % CD] = (x / CD == x % CD) ? 1.f : 0.f;
    __syncthreads();
    // Gram sums over one channel quarter per item: A_ij = sum_c khat_i khat_j E_ij (j < i),
    // P_ij = sum_c q_i khat_j E_ij (j <= i); elementwise operands and the QG, KD, GC records
    for (int it = tid; it < NQ * NP; it += NT) {
        const int p = it % NP, qd = it / NP;
        int i = 0;
        while ((i + 1) * (i + 2) / 2 <= p) ++i;
        const int j = p - i * (i + 1) / 2;
        float sa0 = 0.f, sa1 = 0.f, sp0 = 0.f, sp1 = 0.f;
        const int c0 = qd * (DK / NQ);
#pragma unroll 4
        for (int c = c0; c < c0 + DK / NQ; c += 2) {
            const float e0 = __expf(Gs[i * DK + c] - Gs[j * DK + c]);
            const float e1 = __expf(Gs[i * DK + c + 1] - Gs[j * DK + c + 1]);
            const float k0 = Ks[j * LDK + c] * e0, k1 = Ks[j * LDK + c + 1] * e1;
            sa0 = fmaf(Ks[i * LDK + c], k0, sa0);
            sa1 = fmaf(Ks[i * LDK + c + 1], k1, sa1);
            sp0 = fmaf(Qs[i * LDK + c], k0, sp0);
            sp1 = fmaf(Qs[i * LDK + c + 1], k1, sp1);
        }
        Ap[qd * NP + p] = sa0 + sa1;
        Pp[qd * NP + p] = sp0 + sp1;
    }
    for (int x = tid; x < CD * DK; x += NT) {
        const int i = x / DK, c = x % DK;
        const float G = Gs[i * DK + c], Gl = Gs[(CD - 1) * DK + c];  // G is flat past the last token
        const float gam = __expf(G);
        const float kh = Ks[i * LDK + c];
        Rs[i * LDR + c] = bs[i] * kh * gam;
        rec[R::QG + x] = Qs[i * LDK + c] * gam;
        rec[R::KD + x] = kh * __expf(Gl - G);
        if (i == 0) rec[R::GC + c] = __expf(Gl);
    }
    __syncthreads();
    // the quarters added in a fixed order: A to shared memory, P to the record
    for (int x = tid; x < CD * CD; x += NT) {
        const int i = x / CD, j = x % CD;
        float av = 0.f, pv = 0.f;
        if (j <= i) {
            const int p = i * (i + 1) / 2 + j;
            pv = (Pp[p] + Pp[NP + p]) + (Pp[2 * NP + p] + Pp[3 * NP + p]);
            if (j < i) av = (Ap[p] + Ap[NP + p]) + (Ap[2 * NP + p] + Ap[3 * NP + p]);
        }
        Am[i * LDC + j] = av;
        rec[R::P + x] = pv;
    }
    __syncthreads();
    // (I + Diag(b) A) [W | UP | T] = [Diag(b)(Khat o Gam) | Diag(c) V | I], row by row
    // (Appendix B.2), every column of the right-hand sides at once
    for (int i = 1; i < n; ++i) {
        const float bi = bs[i];
        for (int col = tid; col < NR; col += NT) {
            float sacc = 0.f;
            for (int j = 0; j < i; ++j) sacc = fmaf(Am[i * LDC + j], Rs[j * LDR + col], sacc);
            Rs[i * LDR + col] -= bi * sacc;
        }
        __syncthreads();
    }
    for (int x = tid; x < CD * DK; x += NT) rec[R::W + x] = Rs[(x / DK) * LDR + x % DK];
    for (int x = tid; x < CD * DV; x += NT) {
        const int i = x / DV, c = x % DV;
        rec[R::UP + (c >> 6) * R::kSlice + i * 64 + (c & 63)] = Rs[i * LDR + DK + c];
    }
    if (a.rec_extras) {
        for (int x = tid; x < CD * CD; x += NT) {
            rec[R::XA + x] = Am[(x / CD) * LDC + x % CD];
            rec[R::XT + x] = Rs[(x / CD) * LDR + DK + DV + x % CD];
        }
        for (int x = tid; x < CD * DK; x += NT) rec[R::XG + x] = Gs[x];
    }
}

template <int DK, int DV>
constexpr size_t diag_prep_smem_bytes() {
    return sizeof(float) * (2 * CD * (DK + 1) + CD * DK + CD * (DK + DV + CD + 1) + 8 * NP + CD * (CD + 1) + 2 * CD);
}

template <int DK, int DV>
constexpr size_t diag_state_smem_bytes() {
    using R = DiagRec<DK, DV>;
    return 128 + sizeof(float) * ((size_t)DK * 64 + 2 * (R::kHead + R::kSlice) + 3 * CD * 64) + 64;
}

constexpr int NTS = 512;  // state pass threads: two halves split every contraction

template <int DK, int DV, typename TOut>
__global__ void __launch_bounds__(NTS, 1) diag_state_kernel(FwdArgs a, const float* __restrict__ recs) {
    using R = DiagRec<DK, DV>;
    constexpr uint32_t kHeadBytes = R::kHead * 4, kSliceBytes = R::kSlice * 4;
    constexpr int kStage = R::kHead + R::kSlice;
    constexpr int MH = DK / 32;  // state rows per thread in S' (each half takes every other 16-row block)
    static_assert(kHeadBytes % 16 == 0 && kSliceBytes % 16 == 0, "bulk copy sizes");
    extern __shared__ uint8_t smem_raw[];
    float* sm = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    float* Ss = sm;                     // DK x 64 state slice
    float* stg = Ss + DK * 64;          // 2 stages: [record head | UP slice]
    float* Us = stg + 2 * kStage;       // CD x 64
    float* Pu = Us + CD * 64;           // CD x 64  second half's partial of -W S
    float* Po = Pu + CD * 64;           // CD x 64  second half's partial of QG S
    uint64_t* full = reinterpret_cast<uint64_t*>(Po + CD * 64);

    const int tid = threadIdx.x;
    const int half = tid >> 8, t8 = tid & 255;
    const int sl = blockIdx.x, v0 = sl * 64, h = blockIdx.y, b = blockIdx.z;
    const int T = a.T, H = a.H;
    const int NC = (T + CD - 1) / CD;
    const size_t head = (size_t)b * H + h;
    const size_t sbase = head * DK * DV;
    const float* hrec = recs + head * NC * R::kFloats;
    TOut* o = static_cast<TOut*>(a.o);

    auto request = [&](int c, int st) {
        const uint32_t bar = smem_u32(&full[st]);
        const float* r = hrec + (size_t)c * R::kFloats;
        mbar_expect_tx(bar, kHeadBytes + kSliceBytes);
        bulk_load(smem_u32(stg + st * kStage), r, kHeadBytes, bar);
        bulk_load(smem_u32(stg + st * kStage + R::kHead), r + R::UP + sl * R::kSlice, kSliceBytes, bar);
    };
    if (tid == 0) {
        mbar_init(smem_u32(&full[0]), 1);
        mbar_init(smem_u32(&full[1]), 1);
        fence_mbar_init();
        for (int c = 0; c < min(NC, 2); ++c) request(c, c);
    }
    for (int x = tid; x < DK * 64; x += NTS) {
        const int r = x >> 6, c = x & 63;
        Ss[x] = a.S0 ? a.S0[sbase + (size_t)r * DV + v0 + c] : 0.f;
    }
    __syncthreads();

    const int i = t8 >> 4, cx = 4 * (t8 & 15);  // row (token) and the four columns of this thread
    bool ok = true;
    for (int ci = 0; ci < NC; ++ci) {
        const int st = ci & 1;
        const int t0 = ci * CD, n = min(CD, T - t0);
        const bool got = mbar_wait_bounded(smem_u32(&full[st]), (ci >> 1) & 1, 2000000000ull);
        if (__syncthreads_or(!got)) { ok = false; break; }
        const float* rs = stg + st * kStage;
        if (a.S_chunks) {
            float* dst = a.S_chunks + (head * NC + ci) * DK * DV;
            for (int x = tid; x < DK * 16; x += NTS) {
                const int r = x >> 4, c4 = 4 * (x & 15);
                *reinterpret_cast<float4*>(dst + (size_t)r * DV + v0 + c4) =
                    *reinterpret_cast<const float4*>(Ss + r * 64 + c4);
            }
        }
        // -W S (and QG S when o is wanted; the backward's state recompute wants none) over this
        // half's state rows d in [half DK/2, half DK/2 + DK/2)
        float4 u = make_float4(0.f, 0.f, 0.f, 0.f), oo = u;
        {
            const float* wr = rs + R::W + i * DK;
            const float* qr = rs + R::QG + i * DK;
            const int d0 = half * (DK / 2);
            if (o != nullptr) {
#pragma unroll 8
                for (int d = d0; d < d0 + DK / 2; ++d) {
                    const float w = wr[d], q = qr[d];
                    const float4 s4 = *reinterpret_cast<const float4*>(Ss + d * 64 + cx);
                    u.x = fmaf(-w, s4.x, u.x); u.y = fmaf(-w, s4.y, u.y);
                    u.z = fmaf(-w, s4.z, u.z); u.w = fmaf(-w, s4.w, u.w);
                    oo.x = fmaf(q, s4.x, oo.x); oo.y = fmaf(q, s4.y, oo.y);
                    oo.z = fmaf(q, s4.z, oo.z); oo.w = fmaf(q, s4.w, oo.w);
                }
            } else {
#pragma unroll 8
                for (int d = d0; d < d0 + DK / 2; ++d) {
                    const float w = wr[d];
                    const float4 s4 = *reinterpret_cast<const float4*>(Ss + d * 64 + cx);
                    u.x = fmaf(-w, s4.x, u.x); u.y = fmaf(-w, s4.y, u.y);
                    u.z = fmaf(-w, s4.z, u.z); u.w = fmaf(-w, s4.w, u.w);
                }
            }
        }
        if (half) {
            *reinterpret_cast<float4*>(Pu + i * 64 + cx) = u;
            if (o != nullptr) *reinterpret_cast<float4*>(Po + i * 64 + cx) = oo;
        }
        __syncthreads();
        if (!half) {  // U = UP + both halves of -W S
            const float4 up = *reinterpret_cast<const float4*>(rs + R::kHead + i * 64 + cx);
            const float4 pu = *reinterpret_cast<const float4*>(Pu + i * 64 + cx);
            u = make_float4(up.x + u.x + pu.x, up.y + u.y + pu.y, up.z + u.z + pu.z, up.w + u.w + pu.w);
            *reinterpret_cast<float4*>(Us + i * 64 + cx) = u;
        }
        __syncthreads();
        // O = O1 + P U (row i; the first half adds the second half's O1 partial and stores)
        if (!half && o != nullptr) {
            const float4 po = *reinterpret_cast<const float4*>(Po + i * 64 + cx);
            oo.x += po.x; oo.y += po.y; oo.z += po.z; oo.w += po.w;
            const float* pr = rs + R::P + i * CD;
#pragma unroll
            for (int t = 0; t < CD; ++t) {
                const float p = pr[t];
                const float4 ut = *reinterpret_cast<const float4*>(Us + t * 64 + cx);
                oo.x = fmaf(p, ut.x, oo.x); oo.y = fmaf(p, ut.y, oo.y);
                oo.z = fmaf(p, ut.z, oo.z); oo.w = fmaf(p, ut.w, oo.w);
            }
            if (i < n) {
                TOut* orow = o + tok_index(b, t0 + i, h, T, H) * DV + v0 + cx;
                orow[0] = from_f32<TOut>(oo.x);
                orow[1] = from_f32<TOut>(oo.y);
                orow[2] = from_f32<TOut>(oo.z);
                orow[3] = from_f32<TOut>(oo.w);
            }
        }
        // S' = Diag(GC) S + KD^T U: rows i + 16 (2 m + half) of the state, columns cx .. cx + 3
        {
            float4 acc[MH];
#pragma unroll
            for (int m = 0; m < MH; ++m) {
                const int r = i + 16 * (2 * m + half);
                const float gcr = rs[R::GC + r];
                const float4 s4 = *reinterpret_cast<const float4*>(Ss + r * 64 + cx);
                acc[m] = make_float4(gcr * s4.x, gcr * s4.y, gcr * s4.z, gcr * s4.w);
            }
#pragma unroll
            for (int t = 0; t < CD; ++t) {
                const float4 ut = *reinterpret_cast<const float4*>(Us + t * 64 + cx);
                const float* kd = rs + R::KD + t * DK + i + 16 * half;
#pragma unroll
                for (int m = 0; m < MH; ++m) {
                    const float w = kd[32 * m];
                    acc[m].x = fmaf(w, ut.x, acc[m].x); acc[m].y = fmaf(w, ut.y, acc[m].y);
                    acc[m].z = fmaf(w, ut.z, acc[m].z); acc[m].w = fmaf(w, ut.w, acc[m].w);
                }
            }
#pragma unroll
            for (int m = 0; m < MH; ++m)
                *reinterpret_cast<float4*>(Ss + (i + 16 * (2 * m + half)) * 64 + cx) = acc[m];
        }
        __syncthreads();  // the stage and Us are read: refill the stage
        if (tid == 0 && ci + 2 < NC) request(ci + 2, st);
    }
    if (!ok && tid == 0) atomicOr(&g_diag_error, 1u);
    __syncthreads();
    if (ok && a.S_T) {
        for (int x = tid; x < DK * 16; x += NTS) {
            const int r = x >> 4, c4 = 4 * (x & 15);
            *reinterpret_cast<float4*>(a.S_T + sbase + (size_t)r * DV + v0 + c4) =
                *reinterpret_cast<const float4*>(Ss + r * 64 + c4);
        }
    }
}

template <int DK, int DV, typename Tin, typename TOut>
cudaError_t diag_split_launch(const FwdArgs& a, void* ws, cudaStream_t st) {
    const size_t ps = diag_prep_smem_bytes<DK, DV>(), ss = diag_state_smem_bytes<DK, DV>();
    cudaError_t e = cudaFuncSetAttribute(diag_prep_kernel<DK, DV, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)ps);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(diag_state_kernel<DK, DV, TOut>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ss);
    if (e != cudaSuccess) return e;
    const int NC = (a.T + CD - 1) / CD;
    float* recs = static_cast<float*>(ws);
    diag_prep_kernel<DK, DV, Tin><<<dim3(NC, a.B * a.H), NT, ps, st>>>(a, recs);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    diag_state_kernel<DK, DV, TOut><<<dim3(DV / 64, a.H, a.B), NTS, ss, st>>>(a, recs);
    return cudaGetLastError();
}

template <int DK, typename Tin, typename TOut>
cudaError_t diag_split_dv(const FwdArgs& a, void* ws, cudaStream_t st) {
    return a.Dv == 128 ? diag_split_launch<DK, 128, Tin, TOut>(a, ws, st) : diag_split_launch<DK, 64, Tin, TOut>(a, ws, st);
}
template <int DK, typename Tin>
cudaError_t diag_split_o(const FwdArgs& a, void* ws, cudaStream_t st) {
    return a.out_bf16 ? diag_split_dv<DK, Tin, __nv_bfloat16>(a, ws, st) : diag_split_dv<DK, Tin, float>(a, ws, st);
}

template <int DK, typename Tin, typename TOut>
cudaError_t diag_fwd_launch(const FwdArgs& a, cudaStream_t st) {
    const size_t smem = diag_fwd_smem_bytes<DK>();
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_diag_kernel<DK, Tin, TOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    chunk_fwd_diag_kernel<DK, Tin, TOut><<<dim3(a.Dv / 64, a.H, a.B), NT, smem, st>>>(a);
    return cudaGetLastError();
}

template <int DK, int DV, typename Tin, typename TOut>
cudaError_t diag_bwd_launch(const BwdArgs& a, const FwdArgs& f, const float* recs, cudaStream_t st) {
    const size_t smem = diag_bwd_smem_bytes<DK, DV, Tin>();
    cudaError_t e = cudaFuncSetAttribute(diag_bwd_kernel<DK, DV, Tin, TOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    diag_bwd_kernel<DK, DV, Tin, TOut><<<dim3(DV / 64, a.H, a.B), NT, smem, st>>>(a, f, recs);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t ntok = (size_t)a.B * a.T * a.H;
    diag_finalize_kernel<DK, Tin, TOut><<<(unsigned)((ntok + 7) / 8), 256, 0, st>>>(a, ntok);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t nth = (size_t)a.B * a.H * ((a.T + CD - 1) / CD) * DK;
    diag_dg_kernel<DK><<<(unsigned)((nth + 255) / 256), 256, 0, st>>>(a);
    return cudaGetLastError();
}

template <int DK, typename Tin>
cudaError_t diag_fwd_o(const FwdArgs& a, cudaStream_t st) {
    return a.out_bf16 ? diag_fwd_launch<DK, Tin, __nv_bfloat16>(a, st) : diag_fwd_launch<DK, Tin, float>(a, st);
}
template <int DK, typename Tin, typename TOut>
cudaError_t diag_bwd_dv(const BwdArgs& a, const FwdArgs& f, const float* recs, cudaStream_t st) {
    return a.Dv == 128 ? diag_bwd_launch<DK, 128, Tin, TOut>(a, f, recs, st)
                       : diag_bwd_launch<DK, 64, Tin, TOut>(a, f, recs, st);
}
template <int DK, typename Tin>
cudaError_t diag_bwd_o(const BwdArgs& a, const FwdArgs& f, const float* recs, cudaStream_t st) {
    return a.out_bf16 ? diag_bwd_dv<DK, Tin, __nv_bfloat16>(a, f, recs, st) : diag_bwd_dv<DK, Tin, float>(a, f, recs, st);
}

}  // namespace

int diag_chunk_len() { return CD; }

size_t diag_fwd_workspace(int B, int T, int H, int Dk, int Dv) {
    const size_t NC = ((size_t)T + CD - 1) / CD;
    const size_t rec = Dk == 128 ? (Dv == 128 ? DiagRec<128, 128>::kFloats : DiagRec<128, 64>::kFloats)
                                 : (Dv == 128 ? DiagRec<64, 128>::kFloats : DiagRec<64, 64>::kFloats);
    return (size_t)B * H * NC * rec * sizeof(float);
}

cudaError_t launch_chunk_fwd_diag(const FwdArgs& a, void* ws, size_t ws_bytes, cudaStream_t st) {
    if (ws != nullptr && ws_bytes >= diag_fwd_workspace(a.B, a.T, a.H, a.Dk, a.Dv)) {
        if (a.bf16) return a.Dk == 128 ? diag_split_o<128, __nv_bfloat16>(a, ws, st) : diag_split_o<64, __nv_bfloat16>(a, ws, st);
        return a.Dk == 128 ? diag_split_o<128, float>(a, ws, st) : diag_split_o<64, float>(a, ws, st);
    }
    if (a.bf16) return a.Dk == 128 ? diag_fwd_o<128, __nv_bfloat16>(a, st) : diag_fwd_o<64, __nv_bfloat16>(a, st);
    return a.Dk == 128 ? diag_fwd_o<128, float>(a, st) : diag_fwd_o<64, float>(a, st);
}

cudaError_t diag_take_error(cudaStream_t st, unsigned int* flag) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(flag, g_diag_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_diag_error, &zero, sizeof(unsigned int));
}

// The backward: the forward first writes every 16-token chunk's starting state into
// a.S_chunks (the workspace; the split forward's records go to rec_ws when it is large enough),
// then the reverse pass, the finishing kernel and the dg scan.  The accumulators in `a` must be
// zeroed before this is called.
cudaError_t launch_chunk_bwd_diag(const BwdArgs& a, const float* S0, void* rec_ws, size_t rec_bytes,
                                  cudaStream_t st) {
    FwdArgs f{};
    f.q = a.q;
    f.k = a.k;
    f.v = a.v;
    f.eta = a.eta;
    f.g = a.g;
    f.eps = a.eps;
    f.S0 = S0;
    f.o = nullptr;
    f.S_T = nullptr;
    f.S_chunks = const_cast<float*>(a.S_chunks);
    f.B = a.B;
    f.T = a.T;
    f.H = a.H;
    f.Dk = a.Dk;
    f.Dv = a.Dv;
    f.bf16 = a.bf16;
    f.out_bf16 = false;
    f.rec_extras = true;
    if (rec_ws == nullptr || rec_bytes < diag_fwd_workspace(a.B, a.T, a.H, a.Dk, a.Dv)) return cudaErrorInvalidValue;
    cudaError_t e = launch_chunk_fwd_diag(f, rec_ws, rec_bytes, st);
    if (e != cudaSuccess) return e;
    const float* recs = static_cast<const float*>(rec_ws);
    if (a.bf16)
        return a.Dk == 128 ? diag_bwd_o<128, __nv_bfloat16>(a, f, recs, st) : diag_bwd_o<64, __nv_bfloat16>(a, f, recs, st);
    return a.Dk == 128 ? diag_bwd_o<128, float>(a, f, recs, st) : diag_bwd_o<64, float>(a, f, recs, st);
}

}  // namespace kla
