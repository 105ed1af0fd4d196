// kla_chunk_tc.cu -- chunkwise KLA forward on the 5th-generation tensor cores (sm_100a):
// TMA tile loads, tcgen05.mma with fp32 accumulators in TMEM, fp32 state.
//
// Math ("Kaczmarz Linear Attention", section 4, Propositions 3-4, written on unit keys
// khat = k/r with b = eta r^2/(r^2+eps), c = eta r/(r^2+eps); Appendix B.4 coefficient
// substitution): per chunk of C = 64 tokens with incoming state S (Dk x Dv),
//   P   = Gam o (Q Khat^T)                      (lower incl. diagonal)
//   L   = Diag(b) (Gam^- o Khat Khat^T),  T = (I + L)^{-1}   (forward substitution, B.2)
//   W   = T Diag(b gamma) Khat,  U' = T Diag(c) V,  U = U' - W S          (Eq. 7)
//   O   = Diag(gamma) Q S + P U                                             (Eq. 8)
//   S'  = gamma_last S + (Diag(delta) Khat)^T U,  delta_j = e^{G_last - G_j} (Eq. 9)
//
// Every product is an M = 128 tcgen05 MMA in a transposed form, so one CTA owns a whole
// (b, h) head and TMEM lane = matrix row throughout:
//   Gram   [Q; K] K^T        lane = token (Q rows 0-63, K rows 64-127), col = token
//   SQ     S^T Q^T           lane = dv, col = token
//   W^T    K^T T'^T          lane = dk, col = token        (T' = T Diag(b gamma / r))
//   U^T    V^T T''^T - S^T W^T  lane = dv, col = token     (T'' = T Diag(c))
//   S     += Ktil^T U        lane = dk, col = dv           (Ktil = Diag(delta / r) K)
//   PU     U^T P^T           lane = dv, col = token
// T = (I + L)^{-1} itself is a 64x64 triangular inverse done on CUDA cores (blocked).
// Operands that are computed on chip (P, T', T'', S, U, Ktil) are rounded to bf16 as a
// hi + lo pair and multiplied term by term (the lo x lo term is dropped), which keeps ~16
// significant bits; W enters as a single bf16.  q, k, v are bf16 inputs and exact.
//
// The fp32 master state lives in TMEM (lane = dk, 128 columns): it is kept pre-scaled by the
// coming chunk's gamma_last, and the Ktil^T U MMA accumulates onto it; a bf16 hi/lo copy in
// shared memory is the MMA operand.  One CTA of 256 threads per (b, h): warps w and w + 4
// share TMEM lanes 32 (w % 4) .. + 31 and split the columns of every epilogue.  The chunk loop
// is sequential, with the next chunk's tiles prefetched by TMA into the other stage.  Every
// wait is bounded: on timeout the kernel records an error word and returns after freeing
// TMEM.
#include <cuda.h>

#include "kla_device.cuh"
#include "kla_launch.h"
#include "kla_sm100.cuh"
#include "kla_tc_common.cuh"

namespace kla {

__device__ unsigned int g_tc_error = 0;

namespace {

using namespace sm100;
using namespace tcc;

constexpr int NTHREADS = 256;
constexpr int kIssuer = 128;  // thread that issues the MMAs (warp 4: idle during the scalar prep)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// shared-memory map (offsets from a 1024-aligned base)
constexpr uint32_t OFF_QK = 0;          // 2 stages x 32 KB: [Q;K] rows, two dk blocks
constexpr uint32_t QK_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // 2 stages x 16 KB: V, two dv blocks of [64 x 64]
constexpr uint32_t V_STAGE = 16384;
constexpr uint32_t OFF_SHI = 98304;     // 32 KB: S hi, two dv blocks of [128 dk x 64]
constexpr uint32_t OFF_SLO = 131072;    // 32 KB: S lo
constexpr uint32_t OFF_P = 163840;      // 16 KB: P hi [64 x 64], P lo
constexpr uint32_t OFF_Z = 180224;      // 32 KB: L/T fp32 -> T' T'' hi/lo -> Ktil hi/lo
constexpr uint32_t OFF_MISC = 212992;   // barriers, TMEM slot, per-token scalars
constexpr uint32_t SMEM_BYTES = OFF_MISC + 4096 + 1024;  // + alignment slack

// TMEM columns
constexpr uint32_t TM_G = 0, TM_SQ = 64, TM_W = 128, TM_U = 192, TM_S = 256, TM_PU = 384;

struct Misc {
    uint64_t full[2];
    uint64_t mma;
    uint32_t tmem_base;
    uint32_t pad;
    float G[CH], gam[CH], del[CH], bco[CH], cco[CH], invr[CH], graw[CH], eta[CH];
    float pk[CH];   // e^{-G_j} / r_j, when the chunk's decay range allows the factorised form
    float gsum[2];  // per-warp sums of the next chunk's log-decays
    float grange;   // max |G_j| over the current chunk
};

template <typename TOut>
__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, FwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Misc* ms = reinterpret_cast<Misc*>(sm + OFF_MISC);
    float* Lf = reinterpret_cast<float*>(sm + OFF_Z);  // 64 x LDL fp32
    float* Toff = Lf + 64 * LDL;                          // 6 x 256 fp32
    float* Xs = Toff + 6 * 256;                           // 3 x 256 fp32

    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127;  // TMEM lane owned with the other thread of the pair
    const int ch = tid >> 7;    // which half of an epilogue's columns this thread takes
    const int H = a.H, T = a.T;
    const int NCtot = (T + CH - 1) / CH;
    // one CTA per head (b, h), every chunk [c0, c1) of its sequence in order
    const int head_idx = blockIdx.x;
    const int b = head_idx / H, h = head_idx % H;
    const int c0 = 0, c1 = NCtot;
    const int NC = NCtot;
    const uint32_t sbase = smem_u32(sm);
    const uint32_t bar_full0 = smem_u32(&ms->full[0]);
    const uint32_t bar_mma = smem_u32(&ms->mma);
    const float* S0p = a.S0 ? a.S0 + (size_t)head_idx * DK * DV : nullptr;
    float* STp = a.S_T ? a.S_T + (size_t)head_idx * DK * DV : nullptr;

    if (tid == 0) {
        mbar_init(bar_full0, 1);
        mbar_init(bar_full0 + 8, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ms->tmem_base), 512);
        tmem_relinquish();
    }
    // log-decays of the first chunk (threads 0-63); their sum gives its gamma_last
    float g_next = 0.f, eta_next = 0.f;
    const bool first_valid = NC > 0 && c0 * CH + tid < T;
    if (tid < CH && first_valid) {
        const size_t ti = tok_index(b, c0 * CH + tid, h, T, H);
        g_next = a.g[ti];
        eta_next = a.eta[ti];
    }
    if (warp < 2) {
        const float sg = warp_sum((tid < CH && first_valid) ? g_next : 0.f);
        if ((tid & 31) == 0) ms->gsum[warp] = sg;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms->tmem_base;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

    // Initial state: this thread holds row dk = `row`, columns [64 ch, 64 ch + 64).
    {
        const float g0 = (NC > 0) ? __expf(ms->gsum[0] + ms->gsum[1]) : 1.f;
        float4* sc0 = (a.S_chunks && NC > 0)
                          ? reinterpret_cast<float4*>(a.S_chunks + ((size_t)head_idx * NCtot + c0) * DK * DV +
                                                      (size_t)row * DV + 64 * ch)
                          : nullptr;
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
            float x[32];
            if (S0p) {
                const float4* src = reinterpret_cast<const float4*>(S0p + (size_t)row * DV + 64 * ch + 32 * q2);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 v4 = src[i];
                    x[4 * i] = v4.x; x[4 * i + 1] = v4.y; x[4 * i + 2] = v4.z; x[4 * i + 3] = v4.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = 0.f;
            }
            if (sc0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) sc0[8 * q2 + i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
            }
            st_chunks_split(sm + OFF_SHI + ch * 16384, sm + OFF_SLO + ch * 16384, row, 4 * q2, 4, x);
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] *= g0;
            tmem_st32(tmem + lane_base + TM_S + 64 * ch + 32 * q2, x);
        }
        tmem_st_wait();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    auto issue_loads = [&](int c, int st) {
        const uint32_t bar = bar_full0 + 8 * st;
        const uint32_t qk = sbase + OFF_QK + st * QK_STAGE;
        const uint32_t vv = sbase + OFF_V + st * V_STAGE;
        const int t0 = c * CH;
        mbar_expect_tx(bar, 6 * 8192);
        tma_load_4d(qk, &tm_q, bar, 0, h, t0, b);
        tma_load_4d(qk + 16384, &tm_q, bar, 64, h, t0, b);
        tma_load_4d(qk + 8192, &tm_k, bar, 0, h, t0, b);
        tma_load_4d(qk + 16384 + 8192, &tm_k, bar, 64, h, t0, b);
        tma_load_4d(vv, &tm_v, bar, 0, h, t0, b);
        tma_load_4d(vv + 8192, &tm_v, bar, 64, h, t0, b);
    };
    if (tid == 0 && NC > 0) issue_loads(c0, 0);

    uint32_t mma_phase = 0;
    bool aborted = false;
    int issued = (NC > 0) ? c0 : c0 - 1;  // last chunk whose tiles were requested
    int landed = c0 - 1;                  // last chunk whose tiles were waited for

    // Bounded wait on the MMA barrier shared by the whole CTA; false = give up.
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_bounded(bar_mma, mma_phase, kWaitLimitNs);
        mma_phase ^= 1;
        return !__syncthreads_or(!ok);
    };

    for (int c = c0; c < c1; ++c) {
        const int lc = c - c0;  // chunk index within this CTA's run
        const int st = lc & 1;
        const int t0 = c * CH;
        const int n = min(CH, T - t0);
        uint8_t* qk = sm + OFF_QK + st * QK_STAGE;
        uint8_t* vt = sm + OFF_V + st * V_STAGE;
        const uint32_t qk_a = sbase + OFF_QK + st * QK_STAGE;
        const uint32_t v_a = sbase + OFF_V + st * V_STAGE;

        if (tid < CH) {
            ms->graw[tid] = (tid < n) ? g_next : 0.f;
            ms->eta[tid] = (tid < n) ? eta_next : 0.f;
            if (c + 1 < c1 && (c + 1) * CH + tid < T) {
                const size_t ti = tok_index(b, (c + 1) * CH + tid, h, T, H);
                g_next = a.g[ti];
                eta_next = a.eta[ti];
            }
        }
        if (tid == 0 && c + 1 < c1) issue_loads(c + 1, st ^ 1);
        if (c + 1 < c1) issued = c + 1;
        const bool ok_tma = mbar_wait_bounded(bar_full0 + 8 * st, (lc >> 1) & 1, kWaitLimitNs);
        if (__syncthreads_or(!ok_tma)) { aborted = true; break; }
        landed = c;

        // ---- MMA: Gram = [Q; K] K^T and SQ = S^T Q^T (the scalar prep below overlaps them)
        if (tid == kIssuer) {
            tc_fence_after();
            const uint32_t ig = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
                mma_bf16(tmem + TM_G, smem_desc(qk_a + off, 16, 1024), smem_desc(qk_a + off + 8192, 16, 1024),
                         ig, s > 0);
            }
            const uint32_t isq = idesc_bf16(128, 64, true, false);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t sa = sbase + (part ? OFF_SLO : OFF_SHI);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16(tmem + TM_SQ, smem_desc(sa + s * 2048, 16384, 1024),
                             smem_desc(qk_a + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024), isq, (part | s) > 0);
            }
            mma_commit(bar_mma);
        }

        // key norms and Kaczmarz coefficients (thread 64 + j reads key row j)
        if (tid >= CH && tid < 2 * CH) {
            const int j = tid - CH;
            float r2 = 0.f;
#pragma unroll
            for (int blk = 0; blk < 2; ++blk)
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {  // chunk order rotated by row: no bank conflicts
                    const int cc = (c8 + j) & 7;
                    float f[8];
                    unpack_bf16x8(*reinterpret_cast<const uint4*>(qk + blk * 16384 + 8192 + j * 128 + cc * 16), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) r2 = fmaf(f[e], f[e], r2);
                }
            const KaczCoef cf = kacz_coef(ms->eta[j], r2, a.eps);
            ms->bco[j] = cf.b;
            ms->cco[j] = cf.c;
            ms->invr[j] = cf.inv_r;
        }
        if (warp == 0) {  // inclusive prefix sum of g inside the chunk (2 tokens per lane)
            const int l = tid;
            const float x0 = ms->graw[2 * l], x1 = ms->graw[2 * l + 1];
            float s = x0 + x1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, s, o);
                if (l >= o) s += y;
            }
            const float excl = s - (x0 + x1);
            const float G0 = excl + x0, G1 = excl + x0 + x1;
            ms->G[2 * l] = G0;
            ms->G[2 * l + 1] = G1;
            float gr = fmaxf(fabsf(G0), fabsf(G1));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) gr = fmaxf(gr, __shfl_xor_sync(0xffffffffu, gr, o));
            if (l == 0) ms->grange = gr;
        }
        __syncthreads();
        // e^{G_i - G_j} = gamma_i * e^{-G_j} while every |G_j| < 80 (both factors then stay
        // finite in fp32); otherwise the exact exp of the difference.  Uniform over the CTA.
        const bool factored = ms->grange < 80.f;
        if (tid < CH) {
            ms->gam[tid] = __expf(ms->G[tid]);
            ms->del[tid] = __expf(ms->G[n - 1] - ms->G[tid]);
            ms->pk[tid] = factored ? __expf(-ms->G[tid]) * ms->invr[tid] : 0.f;
        }
        if (!wait_mma()) { aborted = true; break; }
        tc_fence_after();

        // ---- Gram epilogue: P (rows 0-63, hi/lo bf16) and L (rows 64-127, fp32); 32 columns each
        {
            float x[32];
            tmem_ld32(tmem + lane_base + TM_G + 32 * ch, x);
            tmem_ld_wait();
            if (row < CH) {
                const int i = row;
                if (factored) {
                    const float gi = ms->gam[i];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = 32 * ch + e;
                        x[e] = (j <= i) ? gi * x[e] * ms->pk[j] : 0.f;
                    }
                } else {
                    const float Gi = ms->G[i];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = 32 * ch + e;
                        x[e] = (j <= i) ? __expf(Gi - ms->G[j]) * x[e] * ms->invr[j] : 0.f;
                    }
                }
                st_chunks_split(sm + OFF_P, sm + OFF_P + 8192, i, 4 * ch, 4, x);
            } else {
                const int i = row - CH;
                const float bi = ms->bco[i] * ms->invr[i];
                if (factored) {
                    const float bgi = bi * ms->gam[i];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = 32 * ch + e;
                        x[e] = (j < i) ? bgi * x[e] * ms->pk[j] : 0.f;
                    }
                } else {
                    const float Gi = ms->G[i];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = 32 * ch + e;
                        x[e] = (j < i) ? bi * __expf(Gi - ms->G[j]) * x[e] * ms->invr[j] : 0.f;
                    }
                }
                float4* lrow = reinterpret_cast<float4*>(Lf + i * LDL + 32 * ch);
#pragma unroll
                for (int q = 0; q < 8; ++q) lrow[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
            }
        }
        tc_fence_before();
        __syncthreads();
        invert_unit_lower64<NTHREADS>(Lf, Toff, Xs, tid);
        // ---- T' = T Diag(b gamma / r), T'' = T Diag(c): thread -> row tid/4, 16 columns
        {
            const int i = tid >> 2, qq = tid & 3, I = i >> 4;
            float tv[16];
            if (qq <= I) {  // block (I, qq): D_I on the diagonal, Toff below, zero above
                const float* src = (qq == I) ? (Lf + i * LDL + 16 * qq) : (Toff + toff_block(I, qq) * 256 + (i & 15) * 16);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 t4 = *reinterpret_cast<const float4*>(src + 4 * q);
                    tv[4 * q] = t4.x; tv[4 * q + 1] = t4.y; tv[4 * q + 2] = t4.z; tv[4 * q + 3] = t4.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) tv[e] = 0.f;
            }
            __syncthreads();  // T is read; the tiles below overwrite it
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = 16 * qq + e;
                v[e] = tv[e] * (ms->bco[j] * ms->gam[j] * ms->invr[j]);
            }
            st_chunks_split(sm + OFF_Z, sm + OFF_Z + 8192, i, 2 * qq, 2, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = tv[e] * ms->cco[16 * qq + e];
            st_chunks_split(sm + OFF_Z + 16384, sm + OFF_Z + 24576, i, 2 * qq, 2, v);
        }
        fence_proxy_async();
        __syncthreads();

        // ---- MMA: W^T = K^T T'^T and U'^T = V^T T''^T
        if (tid == kIssuer) {
            tc_fence_after();
            const uint32_t iw = idesc_bf16(128, 64, true, false);
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + TM_W, smem_desc(qk_a + 8192 + s * 2048, 16384, 1024),
                             smem_desc(sbase + OFF_Z + part * 8192 + s * 32, 16, 1024), iw, (part | s) > 0);
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + TM_U, smem_desc(v_a + s * 2048, 8192, 1024),
                             smem_desc(sbase + OFF_Z + 16384 + part * 8192 + s * 32, 16, 1024), iw,
                             (part | s) > 0);
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }
        tc_fence_after();
        // ---- W^T to bf16 (over the consumed V stage); Ktil = Diag(delta / r) K hi/lo (over T tiles)
        {
            float x[32];
            tmem_ld32(tmem + lane_base + TM_W + 32 * ch, x);
            tmem_ld_wait();
            st_chunks_bf16(vt, row, 4 * ch, 4, x);
            const int j = tid >> 2, blk = (tid >> 1) & 1, c0 = 4 * (tid & 1);
            const float sc = ms->del[j] * ms->invr[j];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const int cc = c0 + ((c4 + j) & 3);  // rotated by row: no bank conflicts
                float f[8], hi[8], lo[8];
                const uint32_t off = (uint32_t)(j * 128 + cc * 16);  // same swizzle phase: (64 + j) & 7 == j & 7
                unpack_bf16x8(*reinterpret_cast<const uint4*>(qk + blk * 16384 + 8192 + off), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) split_bf16(f[e] * sc, hi[e], lo[e]);
                uint4 uh, ul;
                uh.x = pack_bf16x2(hi[0], hi[1]); uh.y = pack_bf16x2(hi[2], hi[3]);
                uh.z = pack_bf16x2(hi[4], hi[5]); uh.w = pack_bf16x2(hi[6], hi[7]);
                ul.x = pack_bf16x2(lo[0], lo[1]); ul.y = pack_bf16x2(lo[2], lo[3]);
                ul.z = pack_bf16x2(lo[4], lo[5]); ul.w = pack_bf16x2(lo[6], lo[7]);
                *reinterpret_cast<uint4*>(sm + OFF_Z + blk * 8192 + off) = uh;
                *reinterpret_cast<uint4*>(sm + OFF_Z + 16384 + blk * 8192 + off) = ul;
            }
        }
        tc_fence_before();
        fence_proxy_async();
        __syncthreads();

        // ---- MMA: U^T -= S^T W^T
        if (tid == kIssuer) {
            tc_fence_after();
            const uint32_t isw = idesc_bf16(128, 64, true, true, true);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t sa = sbase + (part ? OFF_SLO : OFF_SHI);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16(tmem + TM_U, smem_desc(sa + s * 2048, 16384, 1024),
                             smem_desc(v_a + s * 2048, 8192, 1024), isw, 1);
            }
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }
        tc_fence_after();
        // ---- U^T hi/lo to bf16 over the consumed [Q; K] stage (thread pair = dv row)
        {
            float x[32];
            tmem_ld32(tmem + lane_base + TM_U + 32 * ch, x);
            tmem_ld_wait();
            st_chunks_split(qk, qk + 16384, row, 4 * ch, 4, x);
        }
        if (warp < 2) {  // sum of the next chunk's log-decays (loaded at the top of this chunk)
            const bool valid = (c + 1 < c1) && ((c + 1) * CH + tid < T);
            const float sg = warp_sum(valid ? g_next : 0.f);
            if ((tid & 31) == 0) ms->gsum[warp] = sg;
        }
        tc_fence_before();
        fence_proxy_async();
        __syncthreads();

        // ---- MMA: S += Ktil^T U (N = 128) and PU = U^T P^T
        if (tid == kIssuer) {
            tc_fence_after();
            const uint32_t ids = idesc_bf16(128, 128, true, false);
            const uint32_t ipu = idesc_bf16(128, 64, false, false);
            const uint32_t kt_hi = sbase + OFF_Z, kt_lo = sbase + OFF_Z + 16384;
            const uint32_t u_hi = qk_a, u_lo = qk_a + 16384;
            const uint32_t p_hi = sbase + OFF_P, p_lo = sbase + OFF_P + 8192;
            const uint32_t ka[3] = {kt_hi, kt_hi, kt_lo}, ub[3] = {u_hi, u_lo, u_hi};
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + TM_S, smem_desc(ka[p] + s * 2048, 8192, 1024),
                             smem_desc(ub[p] + s * 32, 16, 1024), ids, 1);
            const uint32_t ua[3] = {u_hi, u_hi, u_lo}, pb[3] = {p_hi, p_lo, p_hi};
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + TM_PU, smem_desc(ua[p] + s * 32, 16, 1024),
                             smem_desc(pb[p] + s * 32, 16, 1024), ipu, (p | s) > 0);
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }
        tc_fence_after();
        // ---- new state to bf16 hi/lo (thread pair = dk row) and outputs (thread pair = dv);
        // TMEM keeps gamma_last(next chunk) * S for the next chunk's accumulation
        {
            const bool has_next = c + 1 < c1;
            const float gN = has_next ? __expf(ms->gsum[0] + ms->gsum[1]) : 1.f;
            float4* scn = (a.S_chunks && has_next)
                              ? reinterpret_cast<float4*>(a.S_chunks + ((size_t)head_idx * NCtot + c + 1) * DK * DV +
                                                          (size_t)row * DV + 64 * ch)
                              : nullptr;
#pragma unroll 1
            for (int q2 = 0; q2 < 2; ++q2) {
                float x[32];
                tmem_ld32(tmem + lane_base + TM_S + 64 * ch + 32 * q2, x);
                tmem_ld_wait();
                st_chunks_split(sm + OFF_SHI + ch * 16384, sm + OFF_SLO + ch * 16384, row, 4 * q2, 4, x);
                if (scn) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        scn[8 * q2 + i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
                }
                if (has_next) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] *= gN;
                    tmem_st32(tmem + lane_base + TM_S + 64 * ch + 32 * q2, x);
                }
            }
            if (has_next) tmem_st_wait();
            if (a.o != nullptr) {
                TOut* o = static_cast<TOut*>(a.o);
                float sq[32], pu[32];
                tmem_ld32(tmem + lane_base + TM_SQ + 32 * ch, sq);
                tmem_ld32(tmem + lane_base + TM_PU + 32 * ch, pu);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int i = 32 * ch + e;
                    if (i < n)
                        o[tok_index(b, t0 + i, h, T, H) * DV + row] = from_f32<TOut>(fmaf(ms->gam[i], sq[e], pu[e]));
                }
            }
        }
        tc_fence_before();
        fence_proxy_async();
        __syncthreads();
    }

    if (aborted) {
        if (tid == 0) atomicOr(&g_tc_error, 1u);
        // let TMA loads that may still be landing in shared memory finish first
        for (int cc = landed + 1; cc <= issued; ++cc)
            (void)mbar_wait_bounded(bar_full0 + 8 * ((cc - c0) & 1), ((cc - c0) >> 1) & 1, kWaitLimitNs);
    } else if (STp) {
        float4* dst = reinterpret_cast<float4*>(STp + (size_t)row * DV + 64 * ch);
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
            float x[32];
            tmem_ld32(tmem + lane_base + TM_S + 64 * ch + 32 * q2, x);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[8 * q2 + i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

// ---------------------------------------------------------------- host side
EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

bool make_map(CUtensorMap* m, const void* base, int B, int T, int H) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc || base == nullptr) return false;
    cuuint64_t dims[4] = {(cuuint64_t)128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)128 * 2, (cuuint64_t)H * 128 * 2, (cuuint64_t)T * H * 128 * 2};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool chunk_fwd_tc_supported(const FwdArgs& a) {
    return a.bf16 && a.Dk == 128 && a.Dv == 128 && a.T > 0 && get_encode_fn() != nullptr;
}

cudaError_t launch_chunk_fwd_tc(const FwdArgs& a, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.B, a.T, a.H) || !make_map(&mk, a.k, a.B, a.T, a.H) ||
        !make_map(&mv, a.v, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    const dim3 grid(a.B * a.H);
    cudaError_t e;
    if (a.out_bf16) {
        e = cudaFuncSetAttribute(chunk_fwd_tc_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        chunk_fwd_tc_kernel<__nv_bfloat16><<<grid, NTHREADS, SMEM_BYTES, st>>>(mq, mk, mv, a);
    } else {
        e = cudaFuncSetAttribute(chunk_fwd_tc_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        chunk_fwd_tc_kernel<float><<<grid, NTHREADS, SMEM_BYTES, st>>>(mq, mk, mv, a);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------
// Scan over segments for the segmented state pass (kla_chunk_split.cu).  The state map of a
// run of chunks is affine, S_end = M S_start + N (the recurrence is linear in the state and
// in the values): pass 1 runs every segment from S = 0 with its values (gives N_s) and from
// S = I with zero values (gives M_s); this scan chains S_{s+1} = M_s S_s + N_s per (b, h) in
// fp32, recording each segment's start; pass 2 runs every segment from its true start.
// ------------------------------------------------------------------------------------
namespace {

constexpr int SCAN_LD = 132;  // padded row of M in shared memory (16-byte rows: vector reads)

// One CTA per (head, 16-column slice of the state): the columns of S evolve independently,
// S_{s+1}[:, cols] = M_s S_s[:, cols] + N_s[:, cols].  M_{s+1} streams into the second of two
// shared-memory buffers (per-thread async copies) and N_{s+1} into registers while step s runs,
// so the chain pays no load latency.  Thread: column tx, rows ty + 16 i (i < 8); the sum over
// k runs in order (k = 0 .. 127), one fma per term.
constexpr int SCAN_W = 16;  // state columns per CTA
constexpr size_t SCAN_SMEM = sizeof(float) * (2 * DK * SCAN_LD + DK * SCAN_W);

__global__ void __launch_bounds__(256) seg_scan_kernel(const float* __restrict__ S0, const float* __restrict__ MN,
                                                       float* __restrict__ Sstart, float* __restrict__ S_T, int BH,
                                                       int nseg) {
    extern __shared__ __align__(16) float scan_sm[];
    float* Mbuf = scan_sm;                   // two 128 x SCAN_LD transitions
    float* Ss = scan_sm + 2 * DK * SCAN_LD;  // 128 x SCAN_W current state columns
    const int head = blockIdx.x, c0 = blockIdx.y * SCAN_W, tid = threadIdx.x;
    const int tx = tid & (SCAN_W - 1), ty = tid >> 4;  // column, row group (rows ty + 16 i)
    const size_t SZ = (size_t)DK * DV;
    auto fetch_M = [&](int sgm) {  // M_sgm (kind 1) into buffer sgm & 1: 16 copies per thread
        const float* M = MN + ((size_t)BH + head) * nseg * SZ + (size_t)sgm * SZ;
        const uint32_t dst = smem_u32(Mbuf + (sgm & 1) * DK * SCAN_LD);
        for (int x = tid; x < DK * DV / 4; x += 256) {
            const int r = (4 * x) / DV, cc = (4 * x) % DV;
            cp_async16(dst + 4 * (uint32_t)(r * SCAN_LD + cc), M + 4 * (size_t)x);
        }
        cp_async_commit();
    };
    auto N_of = [&](int sgm) { return MN + (size_t)head * nseg * SZ + (size_t)sgm * SZ; };  // kind 0
    fetch_M(0);
    for (int x = tid; x < DK * SCAN_W; x += 256) {
        const int r = x / SCAN_W, c = x % SCAN_W;
        Ss[x] = S0 ? S0[head * SZ + (size_t)r * DV + c0 + c] : 0.f;
    }
    float nxt[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) nxt[i] = N_of(0)[(size_t)(ty + 16 * i) * DV + c0 + tx];
    for (int sgm = 0; sgm < nseg; ++sgm) {
        if (sgm + 1 < nseg) {
            fetch_M(sgm + 1);  // its buffer's last reader was step sgm - 1, behind the barrier below
        } else {
            cp_async_commit();  // an empty group keeps the wait below uniform
        }
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = nxt[i];
        if (sgm + 1 < nseg) {
#pragma unroll
            for (int i = 0; i < 8; ++i) nxt[i] = N_of(sgm + 1)[(size_t)(ty + 16 * i) * DV + c0 + tx];
        }
        cp_async_wait<1>();  // this thread's copies of M_sgm have landed
        __syncthreads();     // ... and every thread's; the current columns are in place
        float* out = Sstart + ((size_t)head * nseg + sgm) * SZ;
        for (int x = tid; x < DK * SCAN_W; x += 256) out[(size_t)(x / SCAN_W) * DV + c0 + x % SCAN_W] = Ss[x];
        const float* Ms = Mbuf + (sgm & 1) * DK * SCAN_LD;
#pragma unroll 2
        for (int kk = 0; kk < DK; kk += 4) {
            float bk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) bk[u] = Ss[(kk + u) * SCAN_W + tx];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 m = *reinterpret_cast<const float4*>(Ms + (ty + 16 * i) * SCAN_LD + kk);
                acc[i] = fmaf(m.x, bk[0], acc[i]);
                acc[i] = fmaf(m.y, bk[1], acc[i]);
                acc[i] = fmaf(m.z, bk[2], acc[i]);
                acc[i] = fmaf(m.w, bk[3], acc[i]);
            }
        }
        __syncthreads();  // every read of S and of this M buffer is done
#pragma unroll
        for (int i = 0; i < 8; ++i) Ss[(ty + 16 * i) * SCAN_W + tx] = acc[i];
    }
    __syncthreads();
    if (S_T)
        for (int x = tid; x < DK * SCAN_W; x += 256)
            S_T[head * SZ + (size_t)(x / SCAN_W) * DV + c0 + x % SCAN_W] = Ss[x];
}

}  // namespace

cudaError_t launch_seg_scan(const float* S0, const float* MN, float* Sstart, float* S_T, int BH, int nseg,
                            cudaStream_t st) {
    if (nseg < 1) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(seg_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SCAN_SMEM);
    if (e != cudaSuccess) return e;
    seg_scan_kernel<<<dim3(BH, DV / SCAN_W), 256, SCAN_SMEM, st>>>(S0, MN, Sstart, S_T, BH, nseg);
    return cudaGetLastError();
}

cudaError_t tc_take_error(cudaStream_t st, unsigned int* flag) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(flag, g_tc_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(unsigned int));
}

}  // namespace kla
