// kla_chunk_split.cu -- chunkwise KLA forward split into a chunk-parallel preparation kernel
// and a sequential state pass, both on the 5th-generation tensor cores (sm_100a).
//
// Same math as the fused kernel ("Kaczmarz Linear Attention", section 4, Propositions 3-4,
// Eqs. 7-9, on unit keys khat = k/r with b = eta r^2/(r^2+eps), c = eta r/(r^2+eps)):
//   P   = Gam o (Q Khat^T),   L = Diag(b)(Gam^- o Khat Khat^T),   T = (I + L)^{-1}
//   W   = T Diag(b gamma) Khat,   U' = T Diag(c) V                      (independent of S)
//   U   = U' - W S,   O = Diag(gamma) Q S + P U,   S' = gamma_last S + Ktil^T U,
//   Ktil = Diag(delta) Khat,  delta_j = e^{G_last - G_j}.
// Everything that does not depend on the incoming state -- P, W, T'' = T Diag(c), Ktil and the
// decays -- is computed for all chunks at once by `chunk_prep_kernel` (one CTA per chunk, four
// CTAs per SM) and written to a per-chunk record in the workspace, already in the
// shared-memory image the MMAs read.  `chunk_state_kernel` then walks the chunks of each head in
// order: U' = T'' V (its own V tile; independent of S, so it runs off the chain), U = U' - W S,
// S' and O, with every A operand (S and U as bf16 hi/lo pairs) held in TMEM, so a step is two
// dependent MMA groups and two short epilogues.
//
// State-pass TMEM (lane = dv throughout, 512 columns):
//   [0,128)   S^T master, fp32, pre-scaled by the coming chunk's gamma_last
//   [128,192) S^T hi bf16, [192,256) S^T lo     -- A operand, K = dk
//   [256,320) U^T accumulator fp32 (col = token), [320,384) O1 = S^T Q^T: one N = 128 accumulator
//   [384,416) U^T hi bf16, [416,448) U^T lo     -- A operand, K = token
//   [448,512) O2 = U^T P^T;   o = gamma o O1 + O2
#include <cuda.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <unordered_map>

#include "kla_device.cuh"
#include "kla_launch.h"
#include "kla_sm100.cuh"
#include "kla_tc_common.cuh"

namespace kla {

__device__ unsigned int g_split_error = 0;

namespace {

using namespace sm100;
using namespace tcc;

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s

// The per-chunk record layout (REC_*) is defined in kla_tc_common.cuh.

// =====================================================================================
// Preparation kernel: one chunk per CTA, four CTAs per SM.  Shared memory holds only the
// [Q; K] tile and the MMA operands; every output goes from registers straight to its record.
// U' = T'' V is left to the state pass (the record carries T''), so V is not read here.
// =====================================================================================
constexpr int PT = 256;
constexpr int kPrepIssuer = 128;
constexpr uint32_t P_QK = 0;       // [Q; K] tile (32 KB); after the Gram MMA the inverse's scratch
                                   // (4 KB) over Q block 0, then T' hi/lo over Q
constexpr uint32_t P_Z = 32768;    // L/T fp32 (64 x LDL); then -W staged as [token][dk] tiles
constexpr uint32_t P_MISC = P_Z + 64 * LDL * 4;
constexpr uint32_t P_SMEM = P_MISC + 3072 + 1024;
static_assert(P_MISC % 1024 == 0, "prep scalars alignment");
static_assert(64 * LDL * 4 >= 16384, "-W staging fits over L/T");
constexpr uint32_t PM_G = 0, PM_W = 0;  // TMEM columns (64 allocated); W reuses G's

struct PrepMisc {
    uint64_t full, mma;
    uint32_t tmem_base, pad[3];
    float G[CH], gam[CH], del[CH], bco[CH], cco[CH], invr[CH], eta[CH], pk[CH];
    float wsc[CH];  // b gamma / r: column scale of T'
    float gsum[4], grange;  // the next chunk's g sums (two halves), then the previous chunk's
};
static_assert(sizeof(PrepMisc) <= 3072, "prep scalars");
static_assert(offsetof(PrepMisc, G) % 8 == 0, "float2 access to the per-token scalars");

__global__ void __launch_bounds__(PT, 4)
    chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      FwdArgs a, uint8_t* __restrict__ recs, int cfirst) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PrepMisc* ms = reinterpret_cast<PrepMisc*>(sm + P_MISC);
    float* Lf = reinterpret_cast<float*>(sm + P_Z);  // 64 x LDL fp32: L, then T in place
    float* Xs = reinterpret_cast<float*>(sm + P_QK);   // 1024 floats of scratch for the inverse (over Q)

    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127, ch = tid >> 7;
    const int H = a.H, T = a.T;
    const int NC = (T + CH - 1) / CH;
    const int c = cfirst + blockIdx.x, head = blockIdx.y;
    const int b = head / H, h = head % H;
    const int t0 = c * CH, n = min(CH, T - t0);
    uint8_t* rec = recs + ((size_t)head * NC + c) * REC_BYTES;
    const uint32_t sbase = smem_u32(sm);
    const uint32_t bar_full = smem_u32(&ms->full), bar_mma = smem_u32(&ms->mma);

    // Per-token gates first: their latency, and the in-chunk scan of g and its decays (warp 0),
    // overlap the barrier set-up and the tile loads.  Warp 0 lane l: tokens 2l, 2l + 1 (g zero
    // past the sequence, so G stays flat there); warp 1: eta; warps 2-3 / 4-5: the next /
    // previous chunk's g for its gamma_last.
    float g0 = 0.f, g1 = 0.f, gx = 0.f;
    if (warp == 0) {
        const int l = tid;
        if (2 * l < n) g0 = a.g[tok_index(b, t0 + 2 * l, h, T, H)];
        if (2 * l + 1 < n) g1 = a.g[tok_index(b, t0 + 2 * l + 1, h, T, H)];
    } else if (warp == 1) {
        const int l = tid - 32;
        if (2 * l < n) g0 = a.eta[tok_index(b, t0 + 2 * l, h, T, H)];
        if (2 * l + 1 < n) g1 = a.eta[tok_index(b, t0 + 2 * l + 1, h, T, H)];
    } else if (tid < 2 * CH) {
        const int j = tid - CH;
        if (c + 1 < NC && (c + 1) * CH + j < T) gx = a.g[tok_index(b, (c + 1) * CH + j, h, T, H)];
    } else if (tid < 3 * CH) {  // the previous chunk (always full) for the reverse pass
        if (c > 0) gx = a.g[tok_index(b, (c - 1) * CH + tid - 2 * CH, h, T, H)];
    }
    if (tid == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        mbar_expect_tx(bar_full, 4 * 8192);
        tma_load_4d(sbase + P_QK, &tm_q, bar_full, 0, h, t0, b);
        tma_load_4d(sbase + P_QK + 16384, &tm_q, bar_full, 64, h, t0, b);
        tma_load_4d(sbase + P_QK + 8192, &tm_k, bar_full, 0, h, t0, b);
        tma_load_4d(sbase + P_QK + 24576, &tm_k, bar_full, 64, h, t0, b);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ms->tmem_base), 64);
        tmem_relinquish();
        // inclusive prefix sum G of g inside the chunk, gamma = e^G, delta = e^{G_last - G}
        const int l = tid;
        float sc = g0 + g1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, sc, o);
            if (l >= o) sc += y;
        }
        const float excl = sc - (g0 + g1);
        const float G0 = excl + g0, G1 = excl + g0 + g1;
        const float Glast = __shfl_sync(0xffffffffu, G1, 31);
        float gr = fmaxf(fabsf(G0), fabsf(G1));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) gr = fmaxf(gr, __shfl_xor_sync(0xffffffffu, gr, o));
        const float gm0 = __expf(G0), gm1 = __expf(G1);
        reinterpret_cast<float2*>(ms->G)[l] = make_float2(G0, G1);
        reinterpret_cast<float2*>(ms->gam)[l] = make_float2(gm0, gm1);
        reinterpret_cast<float2*>(ms->del)[l] = make_float2(__expf(Glast - G0), __expf(Glast - G1));
        reinterpret_cast<float2*>(rec + REC_SC)[l] = make_float2(gm0, gm1);
        if (l == 0) ms->grange = gr;
    } else if (warp == 1) {
        reinterpret_cast<float2*>(ms->eta)[tid - 32] = make_float2(g0, g1);
    } else if (tid < 3 * CH) {  // the next (warps 2-3) and previous (warps 4-5) chunks' gamma_last
        const float sg = warp_sum(gx);
        if ((tid & 31) == 0) ms->gsum[warp - 2] = sg;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms->tmem_base;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint8_t* qk = sm + P_QK;
    const uint32_t qk_a = sbase + P_QK;

    bool ok = mbar_wait_bounded(bar_full, 0, kWaitNs);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) atomicOr(&g_split_error, 1u);
        goto done;
    }
    // ---- MMA: Gram = [Q; K] K^T (lane = token; Q rows 0-63, K rows 64-127)
    if (tid == kPrepIssuer) {
        tc_fence_after();
        const uint32_t ig = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
            mma_bf16(tmem + PM_G, smem_desc(qk_a + off, 16, 1024), smem_desc(qk_a + off + 8192, 16, 1024), ig,
                     s > 0);
        }
        mma_commit(bar_mma);
    }
    {
        // e^{G_i - G_j} = gamma_i * e^{-G_j} while every |G_j| < 80; otherwise the exact exp of
        // the difference.  Uniform over the CTA.
        const bool factored = ms->grange < 80.f;
        // key norms and Kaczmarz coefficients: four threads per key row j = tid / 4, thread q of
        // the four summing 32 features (dk block q / 2, logical 16-byte chunks 4 (q & 1) .. + 3 of
        // it, in an order rotated by q / 2 so that the eight lanes of a quarter warp -- rows j and
        // j + 1, whose swizzle phases differ in parity -- hit eight different bank groups)
        {
            const int j = tid >> 2, q = tid & 3;
            const uint8_t* krow = qk + (q >> 1) * 16384 + 8192 + j * 128;
            float ra = 0.f, rb = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int cc = 4 * (q & 1) + ((m + 2 * (q >> 1)) & 3);
                float f[8];
                unpack_bf16x8(*reinterpret_cast<const uint4*>(krow + ((cc ^ (j & 7)) << 4)), f);
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    ra = fmaf(f[e], f[e], ra);
                    rb = fmaf(f[e + 1], f[e + 1], rb);
                }
            }
            float r2 = ra + rb;
            r2 += __shfl_xor_sync(0xffffffffu, r2, 1);
            r2 += __shfl_xor_sync(0xffffffffu, r2, 2);
            if (q == 0) {
                const KaczCoef cf = kacz_coef(ms->eta[j], r2, a.eps);
                ms->bco[j] = cf.b;
                ms->cco[j] = cf.c;
                ms->invr[j] = cf.inv_r;
                ms->pk[j] = factored ? __expf(-ms->G[j]) * cf.inv_r : 0.f;
                ms->wsc[j] = cf.b * ms->gam[j] * cf.inv_r;
            } else if (q == 1 && j < 2) {  // the next / previous chunk's gamma_last
                reinterpret_cast<float*>(rec + REC_SC)[CH + j] = __expf(ms->gsum[2 * j] + ms->gsum[2 * j + 1]);
            }
        }
        ok = mbar_wait_bounded(bar_mma, 0, kWaitNs);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicOr(&g_split_error, 1u);
            goto done;
        }
        tc_fence_after();

        // ---- Gram epilogue: P (rows 0-63, hi/lo bf16, to the record) and L (rows 64-127,
        //      fp32); 32 columns each
        float x[32];
        tmem_ld32(tmem + lane_base + PM_G + 32 * ch, x);
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
            st_chunks_split_global(rec + REC_P, rec + REC_P + 8192, i, 4 * ch, 4, x);
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
    invert_unit_lower64_doubling<PT>(Lf, Xs, tid);
    // ---- T' = T Diag(b gamma / r) over the Q slots of the [Q; K] tile, T'' = T Diag(c) straight
    //      to the record: thread -> row tid/4, 16 columns (T is zero above its diagonal)
    {
        const int i = tid >> 2, qq = tid & 3;
        float tv[16];
        {
            const float* src = Lf + i * LDL + 16 * qq;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 t4 = *reinterpret_cast<const float4*>(src + 4 * q);
                tv[4 * q] = t4.x; tv[4 * q + 1] = t4.y; tv[4 * q + 2] = t4.z; tv[4 * q + 3] = t4.w;
            }
        }
        __syncthreads();  // T is read (and the scratch over Q): T' overwrites Q
        if (a.T_tiles) {
            uint8_t* tt = static_cast<uint8_t*>(a.T_tiles) + ((size_t)head * NC + c) * 16384;
            st_chunks_split_global(tt, tt + 8192, i, 2 * qq, 2, tv);
        }
        float v[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = tv[e] * ms->wsc[16 * qq + e];
        st_chunks_split(sm + P_QK, sm + P_QK + 16384, i, 2 * qq, 2, v);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = tv[e] * ms->cco[16 * qq + e];
        st_chunks_split_global(rec + REC_TPP, rec + REC_TPP + 8192, i, 2 * qq, 2, v);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    // ---- MMA: W^T = K^T T'^T (lane = dk)
    if (tid == kPrepIssuer) {
        tc_fence_after();
        const uint32_t iw = idesc_bf16(128, 64, true, false);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tmem + PM_W, smem_desc(qk_a + 8192 + s * 2048, 16384, 1024),
                         smem_desc(qk_a + part * 16384 + s * 32, 16, 1024), iw, (part | s) > 0);
        mma_commit(bar_mma);
    }
    ok = mbar_wait_bounded(bar_mma, 1, kWaitNs);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) atomicOr(&g_split_error, 1u);
        goto done;
    }
    tc_fence_after();
    {
        // ---- -W (thread = dk column, 32 tokens) transposed to [token][dk] tiles over the consumed
        //      L/T area, then one bulk copy to the record; Ktil hi/lo straight to the record
        float x[32];
        tmem_ld32(tmem + lane_base + PM_W + 32 * ch, x);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = -x[e];
        st_w_tokens_smem(sm + P_Z, row, 32 * ch, x, tid & 31);
        // Ktil row j, dk block blk, logical chunks cq .. cq + 3, in pairs (one 32-byte store
        // each); the pair order alternates with blk so the two blocks' reads of a row (16 KB
        // apart, same banks) do not collide
        const int j = tid >> 2, blk = (tid >> 1) & 1, cq = 4 * (tid & 1);
        const float sc = ms->del[j] * ms->invr[j];
        const uint8_t* krow = qk + blk * 16384 + 8192 + j * 128;  // K row j: swizzle phase (64 + j) & 7 == j & 7
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
            const int c = cq + 2 * ((pp + blk) & 1);
            float f[16];
            unpack_bf16x8(*reinterpret_cast<const uint4*>(krow + ((c ^ (j & 7)) << 4)), f);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(krow + (((c + 1) ^ (j & 7)) << 4)), f + 8);
#pragma unroll
            for (int e = 0; e < 16; ++e) f[e] *= sc;
            uint4 h0, l0, h1, l1;
            split_chunk8(f, h0, l0);
            split_chunk8(f + 8, h1, l1);
            st_pair_sw128_global(rec + REC_KT + blk * 8192, j, c, h0, h1);
            st_pair_sw128_global(rec + REC_KTLO + blk * 8192, j, c, l0, l1);
        }
        fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            bulk_store(rec + REC_W, sbase + P_Z, 16384);
            bulk_commit();
            bulk_wait_read();
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

// =====================================================================================
// Preparation kernel with diagonal gating (per-key-channel decays, "Kaczmarz Linear
// Attention", Appendix B.5), on the tensor cores: one 64-token chunk per CTA, two CTAs per SM.
// With G_t the in-chunk prefix of the log-decays (a vector over channels) the pairwise factor
// exp(G_i - G_j) sits inside the channel sums of the Gram and score tiles, so it is split per
// channel around a reference R = (max_t G_t + min_t G_t) / 2:
//   [Q; Khat] o exp(G - R)  times  (Khat o exp(R - G))^T   (hi/lo bf16, three products)
// gives every entry j <= i exactly; each factor is at most exp(range / 2), so a channel whose
// in-chunk range reaches 160 takes the exact product on the CUDA cores instead (the entries
// above the diagonal, which can overflow, are masked away).  W = T Diag(b) (Khat o Gam)
// (Gam_t = exp(G_t) <= 1) is a tensor-core product as for scalar gating, and T'' = T Diag(c)
// goes to the record for the state pass's U' = T'' V; the record adds Q o Gam for the state
// pass's O1 product and the chunk's own and the next chunk's Gam_last per channel for its
// rescale.
// =====================================================================================
constexpr uint32_t PD_K = 0;         // raw K tile (16 KB, TMA: two 64-dk blocks)
constexpr uint32_t PD_C = 16384;     // G fp32 [64][128] (32 KB); then L/T + scratch; then T' hi/lo
constexpr uint32_t PD_D = 49152;     // next chunk's g (32 KB); then one dk half of the Gram operands
                                     // (X hi/lo 32 KB, Y hi/lo 16 KB); then K o Gam hi/lo (32 KB)
constexpr uint32_t PD_MISC = PD_D + 49152;
constexpr uint32_t PD_SMEM = PD_MISC + 5120 + 1024;
constexpr uint32_t PDM_G = 0, PDM_W = 64;  // TMEM columns (128 allocated)
constexpr float kDiagRange = 160.f;  // in-chunk range of G above which the Gram is formed exactly

struct PrepDiagMisc {
    uint64_t full, nextg, mma;
    uint32_t tmem_base, wide;
    float bco[CH], cco[CH], invr[CH], eta[CH];
    float R[DK], Gl[DK], gh[DK];
    float mx[2][DK], mn[2][DK];
};
static_assert(sizeof(PrepDiagMisc) <= 5120, "prep scalars");

// Eight consecutive channels [d0, d0 + 8) of token row t of the raw K tile, times s.
__device__ __forceinline__ void k_chunk8(const uint8_t* ktile, int t, int d0, float s, float* f) {
    unpack_bf16x8(*reinterpret_cast<const uint4*>(ktile + (d0 >> 6) * 8192 + sw128_off(t, (d0 & 63) >> 3)), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] *= s;
}
// Eight consecutive channels of q at token t of (b, h) (zeros past the sequence).
__device__ __forceinline__ void q_chunk8(const FwdArgs& a, int b, int t, int h, int d0, float* f) {
    if (t < a.T) {
        const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
        unpack_bf16x8(*reinterpret_cast<const uint4*>(q + tok_index(b, t, h, a.T, a.H) * DK + d0), f);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.f;
    }
}

__global__ void __launch_bounds__(PT, 2)
    chunk_prep_diag_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_g, FwdArgs a,
                           uint8_t* __restrict__ recs, int cfirst) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PrepDiagMisc* ms = reinterpret_cast<PrepDiagMisc*>(sm + PD_MISC);
    float* Gs = reinterpret_cast<float*>(sm + PD_C);  // [64][DK]
    float* Lf = Gs;                                     // later: L, then T in place
    float* Xs = Lf + 64 * LDL;                          // 1024 floats of scratch for the inverse

    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127, ch = tid >> 7;
    const int H = a.H, T = a.T;
    const int NC = (T + CH - 1) / CH;
    const int c = cfirst + blockIdx.x, head = blockIdx.y;
    const int b = head / H, h = head % H;
    const int t0 = c * CH, n = min(CH, T - t0);
    const bool has_next = c + 1 < NC;
    uint8_t* rec = recs + ((size_t)head * NC + c) * REC_BYTES_D;
    const uint32_t sbase = smem_u32(sm);
    const uint32_t bar_full = smem_u32(&ms->full), bar_next = smem_u32(&ms->nextg),
                   bar_mma = smem_u32(&ms->mma);

    const float eta_own = (tid < n) ? a.eta[tok_index(b, t0 + tid, h, T, H)] : 0.f;
    // this thread's q chunks, loaded first so that their latency overlaps the set-up: rows tq and
    // tq + 32, 16-byte chunk cq of each 64-channel half (the X operands' Q rows and the record's
    // Q o Gam take the same ones)
    const int tq = tid >> 3, cq = tid & 7;
    uint4 qv[2][2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int t = t0 + tq + 32 * k;
            qv[hf][k] = t < T ? *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                                                 tok_index(b, t, h, T, H) * DK + 64 * hf + 8 * cq)
                              : make_uint4(0u, 0u, 0u, 0u);
        }
    if (tid == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar_next, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        mbar_expect_tx(bar_full, 16384 + 32768);
        tma_load_4d(sbase + PD_K, &tm_k, bar_full, 0, h, t0, b);
        tma_load_4d(sbase + PD_K + 8192, &tm_k, bar_full, 64, h, t0, b);
        tma_load_4d(sbase + PD_C, &tm_g, bar_full, 0, h, t0, b);
        if (has_next) {
            mbar_expect_tx(bar_next, 32768);
            tma_load_4d(sbase + PD_D, &tm_g, bar_next, 0, h, t0 + CH, b);
        }
        ms->wide = 0u;
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ms->tmem_base), 128);
        tmem_relinquish();
    }
    if (tid < CH) ms->eta[tid] = eta_own;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms->tmem_base;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    bool aborted = false, next_pending = has_next;
    int mma_phase = 0;

    do {
        if (__syncthreads_or(!mbar_wait_bounded(bar_full, 0, kWaitNs))) { aborted = true; break; }
        // ---- key norms and coefficients: four threads per key row (as for scalar gating)
        {
            const int j = tid >> 2, q = tid & 3;
            const uint8_t* krow = sm + PD_K + (q >> 1) * 8192 + j * 128;
            float ra = 0.f, rb = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int cc = 4 * (q & 1) + ((m + 2 * (q >> 1)) & 3);
                float f[8];
                unpack_bf16x8(*reinterpret_cast<const uint4*>(krow + ((cc ^ (j & 7)) << 4)), f);
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    ra = fmaf(f[e], f[e], ra);
                    rb = fmaf(f[e + 1], f[e + 1], rb);
                }
            }
            float r2 = ra + rb;
            r2 += __shfl_xor_sync(0xffffffffu, r2, 1);
            r2 += __shfl_xor_sync(0xffffffffu, r2, 2);
            if (q == 0) {
                const KaczCoef cf = kacz_coef(ms->eta[j], r2, a.eps);
                ms->bco[j] = cf.b;
                ms->cco[j] = cf.c;
                ms->invr[j] = cf.inv_r;
            }
        }
        // ---- per-channel prefix sums of g over the chunk: thread (channel d, half hf) scans 32
        //      tokens in registers; the second half then adds the first half's total
        {
            const int d = tid & 127, hf = tid >> 7;
            float gv[32];
#pragma unroll
            for (int t = 0; t < 32; ++t) gv[t] = Gs[(32 * hf + t) * DK + d];
#pragma unroll
            for (int t = 1; t < 32; ++t) gv[t] += gv[t - 1];
            if (hf == 0) ms->gh[d] = gv[31];
            __syncthreads();
            const float off = hf ? ms->gh[d] : 0.f;
            float mx = -INFINITY, mn = INFINITY;
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                gv[t] += off;
                Gs[(32 * hf + t) * DK + d] = gv[t];
                mx = fmaxf(mx, gv[t]);
                mn = fminf(mn, gv[t]);
            }
            ms->mx[hf][d] = mx;
            ms->mn[hf][d] = mn;
            __syncthreads();
            if (hf == 0) {
                const float hi = fmaxf(ms->mx[0][d], ms->mx[1][d]), lo = fminf(ms->mn[0][d], ms->mn[1][d]);
                ms->R[d] = 0.5f * (hi + lo);
                if (!(hi - lo < kDiagRange)) atomicOr(&ms->wide, 1u);
            } else {
                ms->Gl[d] = gv[31];  // G is flat past the last token
                reinterpret_cast<float*>(rec + REC_GL)[d] = __expf(gv[31]);
            }
        }
        // ---- the next chunk's Gam_last per channel (the state pass's rescale)
        if (has_next) {
            if (__syncthreads_or(!mbar_wait_bounded(bar_next, 0, kWaitNs))) { aborted = true; break; }
            next_pending = false;
            const int d = tid & 127, hf = tid >> 7;
            const float* gn = reinterpret_cast<const float*>(sm + PD_D);
            float s = 0.f;
#pragma unroll 8
            for (int t = 0; t < 32; ++t) s += gn[(32 * hf + t) * DK + d];
            if (hf == 1) ms->gh[d] = s;
            __syncthreads();
            if (hf == 0) reinterpret_cast<float*>(rec + REC_SC)[d] = __expf(s + ms->gh[d]);
        } else if (tid < DK) {
            reinterpret_cast<float*>(rec + REC_SC)[tid] = 1.f;
        }
        __syncthreads();
        const bool wide = ms->wide != 0u;
        const float* Rr = ms->R;

        // ---- Gram and scores, one dk half at a time; the record's Q o Gam and Ktil hi/lo for the
        //      same half while its products run
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            uint8_t* Xh = sm + PD_D;
            uint8_t* Xl = Xh + 16384;
            uint8_t* Yh = Xh + 32768;
            uint8_t* Yl = Xh + 40960;
            if (!wide) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int r = tq + 32 * k, i = r & 63, d0 = 64 * hf + 8 * cq;
                    float f[8];
                    if (k < 2) unpack_bf16x8(qv[hf][k & 1], f);
                    else k_chunk8(sm + PD_K, i, d0, ms->invr[i], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] *= __expf(Gs[i * DK + d0 + e] - Rr[d0 + e]);
                    uint4 uh, ul;
                    split_chunk8(f, uh, ul);
                    *reinterpret_cast<uint4*>(Xh + sw128_off(r, cq)) = uh;
                    *reinterpret_cast<uint4*>(Xl + sw128_off(r, cq)) = ul;
                }
                for (int u = tid; u < 64 * 8; u += PT) {
                    const int j = u >> 3, cc = u & 7, d0 = 64 * hf + 8 * cc;
                    float f[8];
                    k_chunk8(sm + PD_K, j, d0, ms->invr[j], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] *= __expf(Rr[d0 + e] - Gs[j * DK + d0 + e]);
                    uint4 uh, ul;
                    split_chunk8(f, uh, ul);
                    *reinterpret_cast<uint4*>(Yh + sw128_off(j, cc)) = uh;
                    *reinterpret_cast<uint4*>(Yl + sw128_off(j, cc)) = ul;
                }
                fence_proxy_async();
                tc_fence_before();
                __syncthreads();
                if (tid == kPrepIssuer) {
                    tc_fence_after();
                    const uint32_t ig = idesc_bf16(128, 64, false, false);
                    const uint32_t xa[3] = {sbase + PD_D, sbase + PD_D, sbase + PD_D + 16384};
                    const uint32_t yb[3] = {sbase + PD_D + 32768, sbase + PD_D + 40960, sbase + PD_D + 32768};
#pragma unroll
                    for (int p = 0; p < 3; ++p)
#pragma unroll
                        for (int s = 0; s < 4; ++s)
                            mma_bf16(tmem + PDM_G, smem_desc(xa[p] + s * 32, 16, 1024), smem_desc(yb[p] + s * 32, 16, 1024),
                                     ig, (hf | p | s) > 0);
                    mma_commit(bar_mma);
                }
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = tq + 32 * k, cc = cq, d0 = 64 * hf + 8 * cc;
                float f[8], kq[8];
                unpack_bf16x8(qv[hf][k], f);
                k_chunk8(sm + PD_K, t, d0, ms->invr[t], kq);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float G = Gs[t * DK + d0 + e];
                    f[e] *= __expf(G);
                    kq[e] *= __expf(ms->Gl[d0 + e] - G);
                }
                uint4 uq;
                uq.x = pack_bf16x2(f[0], f[1]); uq.y = pack_bf16x2(f[2], f[3]);
                uq.z = pack_bf16x2(f[4], f[5]); uq.w = pack_bf16x2(f[6], f[7]);
                *reinterpret_cast<uint4*>(rec + REC_QG + hf * 8192 + sw128_off(t, cc)) = uq;
                uint4 uh, ul;
                split_chunk8(kq, uh, ul);
                *reinterpret_cast<uint4*>(rec + REC_KT + hf * 8192 + sw128_off(t, cc)) = uh;
                *reinterpret_cast<uint4*>(rec + REC_KTLO + hf * 8192 + sw128_off(t, cc)) = ul;
            }
            if (!wide) {
                const bool okm = mbar_wait_bounded(bar_mma, mma_phase & 1, kWaitNs);
                ++mma_phase;
                if (__syncthreads_or(!okm)) { aborted = true; break; }
                tc_fence_after();
            }
        }
        if (aborted) break;
        // ---- a chunk too wide for the factored products: the Gram and scores exactly (row of
        //      [Q; Khat] = TMEM lane, 32 key columns a thread)
        if (wide) {
            const int i = row & 63;
            float acc[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = 0.f;
            for (int d0 = 0; d0 < DK; d0 += 8) {
                float x[8], gi[8];
                if (row < 64) q_chunk8(a, b, t0 + i, h, d0, x);
                else k_chunk8(sm + PD_K, i, d0, ms->invr[i], x);
#pragma unroll
                for (int e = 0; e < 8; ++e) gi[e] = Gs[i * DK + d0 + e];
                for (int e2 = 0; e2 < 32; ++e2) {
                    const int j = 32 * ch + e2;
                    float kj[8];
                    k_chunk8(sm + PD_K, j, d0, ms->invr[j], kj);
                    float s = acc[e2];
#pragma unroll
                    for (int e = 0; e < 8; ++e) s = fmaf(x[e] * kj[e], __expf(gi[e] - Gs[j * DK + d0 + e]), s);
                    acc[e2] = s;
                }
            }
            tmem_st32(tmem + lane_base + PDM_G + 32 * ch, acc);
            tmem_st_wait();
        }
        // ---- K o Gam hi/lo (the A operand of W^T), [token][dk] blocks like the raw K tile
        for (int u = tid; u < 64 * 16; u += PT) {
            const int t = u >> 4, c16 = u & 15, d0 = 8 * c16;
            float f[8];
            k_chunk8(sm + PD_K, t, d0, ms->invr[t], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] *= __expf(Gs[t * DK + d0 + e]);
            uint4 uh, ul;
            split_chunk8(f, uh, ul);
            const uint32_t o = (c16 >> 3) * 8192 + sw128_off(t, c16 & 7);
            *reinterpret_cast<uint4*>(sm + PD_D + o) = uh;
            *reinterpret_cast<uint4*>(sm + PD_D + 16384 + o) = ul;
        }
        tc_fence_before();
        __syncthreads();  // G is no longer read: L takes its place
        tc_fence_after();
        // ---- Gram epilogue: P (rows 0-63, hi/lo to the record) and L (rows 64-127, fp32)
        {
            float x[32];
            tmem_ld32(tmem + lane_base + PDM_G + 32 * ch, x);
            tmem_ld_wait();
            if (row < CH) {
                const int i = row;
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = (32 * ch + e <= i) ? x[e] : 0.f;
                st_chunks_split_global(rec + REC_P, rec + REC_P + 8192, i, 4 * ch, 4, x);
            } else {
                const int i = row - CH;
                const float bi = ms->bco[i];
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = (32 * ch + e < i) ? bi * x[e] : 0.f;
                float4* lrow = reinterpret_cast<float4*>(Lf + i * LDL + 32 * ch);
#pragma unroll
                for (int q = 0; q < 8; ++q) lrow[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
            }
        }
        tc_fence_before();
        __syncthreads();
        invert_unit_lower64_doubling<PT>(Lf, Xs, tid);
        // ---- T' = T Diag(b) as bf16 hi/lo over the L/T area, T'' = T Diag(c) straight to the record
        {
            const int i = tid >> 2, qq = tid & 3;
            float tv[16];
            {
                const float* src = Lf + i * LDL + 16 * qq;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 t4 = *reinterpret_cast<const float4*>(src + 4 * q);
                    tv[4 * q] = t4.x; tv[4 * q + 1] = t4.y; tv[4 * q + 2] = t4.z; tv[4 * q + 3] = t4.w;
                }
            }
            __syncthreads();  // T is read; T' overwrites it
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = tv[e] * ms->bco[16 * qq + e];
            st_chunks_split(sm + PD_C, sm + PD_C + 8192, i, 2 * qq, 2, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = tv[e] * ms->cco[16 * qq + e];
            st_chunks_split_global(rec + REC_TPP, rec + REC_TPP + 8192, i, 2 * qq, 2, v);
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        // ---- MMA: W^T = (K o Gam)^T T'^T (lane = dk; products hi.hi, hi.lo, lo.hi)
        if (tid == kPrepIssuer) {
            tc_fence_after();
            const uint32_t iw = idesc_bf16(128, 64, true, false);
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16(tmem + PDM_W, smem_desc(sbase + PD_D + (p == 2 ? 16384 : 0) + s * 2048, 8192, 1024),
                             smem_desc(sbase + PD_C + (p == 1 ? 8192 : 0) + s * 32, 16, 1024), iw, (p | s) > 0);
            mma_commit(bar_mma);
        }
        {
            const bool okm = mbar_wait_bounded(bar_mma, mma_phase & 1, kWaitNs);
            ++mma_phase;
            if (__syncthreads_or(!okm)) { aborted = true; break; }
        }
        tc_fence_after();
        // ---- -W transposed to [token][dk] over the consumed K o Gam tiles (one bulk copy to the
        //      record)
        {
            float x[32];
            tmem_ld32(tmem + lane_base + PDM_W + 32 * ch, x);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = -x[e];
            st_w_tokens_smem(sm + PD_D, row, 32 * ch, x, tid & 31);
            fence_proxy_async();
            __syncthreads();
            if (tid == 0) {
                bulk_store(rec + REC_W, sbase + PD_D, 16384);
                bulk_commit();
                bulk_wait_read();
            }
        }
    } while (false);
    if (aborted && tid == 0) {
        atomicOr(&g_split_error, 1u);
        // copies still in flight land before the block exits
        if (next_pending) (void)mbar_wait_bounded(bar_next, 0, kWaitNs);
        (void)mbar_wait_bounded(bar_full, 0, kWaitNs);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// =====================================================================================
// State pass: one CTA per (b, h) [segment, kind], chunks in order.  Warp-specialised:
// warps 0-7 run the epilogues (thread pair = one TMEM lane = one dv column, the two threads
// splitting the columns), warp 8 issues the MMAs, warp 9 moves the stages in and the outputs
// out.  They meet on mbarriers:
//   issuer -> epilogue: bar_u (U^T ready in TMEM), bar_s (S^T updated), bar_o (O1, O2 ready)
//   epilogue -> issuer: s_ready[2], u_ready[2] (each half of the S, U operands written),
//                       o_read (O1 and O2 read out of TMEM)
//   epilogue -> loader: o_free (the o tile staged)
// bar_o and o_free, which the loader also waits on, come one per stage: a phase of either
// cannot come round again before the loader has refilled that stage, so the loader's parity
// waits never alias even when it runs late.
// An MMA issue blocks its thread while the tensor pipe drains, so no epilogue work sits on the
// issuing warp; and the S and U operands are released in halves, so the first K steps of the
// MMA that consumes them run while the epilogue finishes the second half.  Per chunk c:
//   issuer    U'(c) = V^T T''^T | [U | O1 hi](c) [2 halves] | O1 lo(c) | S(c) [2 halves] O2(c)
//   epilogue  U epi(c) -> S hi/lo(c+1) -> master rescale -> O epi(c) (O1 zeroed once read)
//   loader    refill of chunk c's stage with chunk c + 2 (part A: -W, Q, P, T'', V once chunk
//             c's MMAs are done; part B: Ktil and scalars once the o tile has left by TMA store)
// U'(c) accumulates into U's columns ahead of the S-dependent product, so it runs while the
// previous chunk's state epilogue does; O1, which shares that N = 128 accumulator, is zeroed by
// the output epilogue after reading it so that the [U | O1] product can always accumulate.
// =====================================================================================
constexpr int ST = 320;
constexpr int kIssuerWarp = 8, kLoaderWarp = 9;
constexpr uint32_t S_STAGE = 114688;  // Q 16 KB + the record's tiles (80 KB) + V 16 KB
// SO_WQ: [-W block 0 | Q block 0 | -W block 1 | Q block 1], 8 KB each ([64 tokens x 64 dk]),
// so that one K-major descriptor over 128 rows reads -W then Q for the same 16 dk: the U and
// O1 products share their A operand (S^T) and run as N = 128 MMAs.  The o tile is staged over
// Ktil (32 KB) once the chunk's MMAs are done.
constexpr uint32_t SO_WQ = 0, SO_KT = 32768, SO_KTLO = 49152, SO_P = 65536, SO_PLO = 73728, SO_TPP = 81920,
                   SO_V = 98304;
static_assert(SO_KT == REC_KT + 16384 && SO_KTLO == REC_KTLO + 16384 && SO_P == REC_P + 16384 &&
                  SO_TPP == REC_TPP + 16384,
              "stage mirrors the record");
static_assert(S_STAGE - SO_KT == 32768 + 16384 + 16384 + 16384, "Ktil, P, T'', V fill the rest of the stage");
constexpr uint32_t S_SC = 2 * S_STAGE;  // 2 x 512 B record scalars
constexpr uint32_t S_MISC = S_SC + 2 * REC_SCB;
constexpr uint32_t S_GL0 = S_MISC + 256;  // diagonal gating: the first chunk's Gam_last[128]
constexpr uint32_t S_SMEM = S_GL0 + 512 + 1024;
constexpr uint32_t TM_S = 0, TM_SH = 128, TM_SL = 192, TM_U = 256, TM_O1 = 320, TM_UH = 384, TM_UL = 416,
                   TM_O2 = 448;
static_assert(TM_O1 == TM_U + 64, "U and O1 are one N = 128 accumulator");

struct StateMisc {
    uint64_t full_a[2], full_b[2];                // the two parts of each stage (TMA / bulk bytes)
    uint64_t bar_u, bar_s, bar_o[2];              // tcgen05.commit arrivals (bar_o per stage)
    uint64_t s_ready[2], u_ready[2], o_free[2];   // one arrival per epilogue warp (o_free per stage)
    uint64_t o_read;                              // O1 and O2 read out of TMEM (one arrival per warp)
    uint32_t tmem_base, abort;
    float gsum[2];
};
static_assert(sizeof(StateMisc) <= 256, "state scalars");

__device__ __forceinline__ void tma_store_4d(const void* tmap, uint32_t src, int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(tmap)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
template <typename TOut, bool DIAG>
__global__ void __launch_bounds__(ST, 1)
    chunk_state_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o, FwdArgs a, const uint8_t* __restrict__ recs) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    StateMisc* ms = reinterpret_cast<StateMisc*>(sm + S_MISC);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = tid & 127;        // TMEM lane = dv (epilogue warps)
    const int ch = (tid >> 7) & 1;    // half of every epilogue's columns
    const int H = a.H, T = a.T;
    const int NCtot = (T + CH - 1) / CH;
    const int nseg = a.nseg > 1 ? a.nseg : 1;
    const bool segmented = a.nseg > 1;
    const int segc = a.seg_chunks > 0 ? a.seg_chunks : NCtot;  // chunks of this run (segment or slab)
    const int head_idx = blockIdx.x / nseg, seg = blockIdx.x % nseg;
    const int BH = gridDim.x / nseg;
    const int b = head_idx / H, h = head_idx % H;
    const bool ident = blockIdx.y == 1;  // transition pass: identity start, zero values, no outputs
    const int c0 = (segmented ? 0 : a.chunk0) + seg * segc, c1 = min(NCtot, c0 + segc);
    const int NC = c1 > c0 ? c1 - c0 : 0;
    const uint32_t sbase = smem_u32(sm);
    const uint32_t full_a0 = smem_u32(&ms->full_a[0]), full_b0 = smem_u32(&ms->full_b[0]);
    const uint32_t bar_u = smem_u32(&ms->bar_u), bar_s = smem_u32(&ms->bar_s), bar_o0 = smem_u32(&ms->bar_o[0]);
    const uint32_t s_ready0 = smem_u32(&ms->s_ready[0]), u_ready0 = smem_u32(&ms->u_ready[0]),
                   o_free0 = smem_u32(&ms->o_free[0]), o_read = smem_u32(&ms->o_read);
    const float* S0p = (a.S0 && !ident)
                           ? a.S0 + (size_t)(segmented ? head_idx * nseg + seg : head_idx) * DK * DV
                           : nullptr;
    float* STp = a.S_T ? a.S_T + (size_t)(segmented ? ((size_t)blockIdx.y * BH + head_idx) * nseg + seg : head_idx) *
                                     DK * DV
                       : nullptr;
    float* Sc = (a.S_chunks && !ident) ? a.S_chunks + (size_t)head_idx * NCtot * DK * DV : nullptr;
    uint8_t* Stl = (a.S_tiles && !ident) ? static_cast<uint8_t*>(a.S_tiles) + (size_t)head_idx * NCtot * 65536 : nullptr;
    uint8_t* Utl = (a.U_tiles && !ident) ? static_cast<uint8_t*>(a.U_tiles) + (size_t)head_idx * NCtot * 32768 : nullptr;
    const bool write_o = !ident && a.o != nullptr;
    // Without outputs (the transition pass of the segmented mode) Q, P and the O products are not
    // needed; with zero values (its identity kind) neither is U'.
    const bool need_vals = !ident;
    // Diagonal gating: Q o Gam comes with the record (the output needs no per-token gamma), the
    // master state's rescale is per key channel, and records are longer.
    constexpr bool diag = DIAG;
    const size_t rstride = diag ? REC_BYTES_D : REC_BYTES;
    const float* gl0 = reinterpret_cast<const float*>(sm + S_GL0);

    if (tid == 0) {
        mbar_init(full_a0, 1);
        mbar_init(full_a0 + 8, 1);
        mbar_init(full_b0, 1);
        mbar_init(full_b0 + 8, 1);
        mbar_init(bar_u, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_o0, 1);
        mbar_init(bar_o0 + 8, 1);
        mbar_init(s_ready0, 8);
        mbar_init(s_ready0 + 8, 8);
        mbar_init(u_ready0, 8);
        mbar_init(u_ready0 + 8, 8);
        mbar_init(o_free0, 8);
        mbar_init(o_free0 + 8, 8);
        mbar_init(o_read, 8);
        ms->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ms->tmem_base), 512);
        tmem_relinquish();
    }
    if (diag) {  // Gam_last of the first chunk, per key channel, from its record
        if (tid < DK)
            reinterpret_cast<float*>(sm + S_GL0)[tid] =
                NC > 0 ? reinterpret_cast<const float*>(recs + ((size_t)head_idx * NCtot + c0) * rstride + REC_GL)[tid]
                       : 1.f;
    } else if (warp < 2) {  // gamma_last of the first chunk
        const bool live = NC > 0 && c0 * CH + tid < T;
        const float gv = live ? a.g[tok_index(b, c0 * CH + tid, h, T, H)] : 0.f;
        const float sg = warp_sum(gv);
        if (lane == 0) ms->gsum[warp] = sg;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms->tmem_base;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

    bool aborted = false;
    if (warp == kLoaderWarp) {
        // ================================ loader ================================
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            if (need_vals) prefetch_tmap(&tm_v);
            if (write_o) prefetch_tmap(&tm_o);
            // Part A of chunk c (-W, Q, P, T'', V: the operands of its first products) can land as soon
            // as chunk c - 2's MMAs are done; part B (Ktil, needed from the S product on, and the
            // scalars, read by the epilogues up to chunk c - 2's o tile) only after that tile,
            // staged over Ktil, has left by TMA store.
            const uint32_t a_bytes = 16384 + (write_o ? 32768 : 0) + (need_vals ? 32768 : 0);
            const uint32_t b_bytes = 32768 + REC_SCB;
            auto load_a = [&](int c, int st) {
                const uint32_t bar = full_a0 + 8 * st;
                const uint32_t base = sbase + st * S_STAGE;
                const uint8_t* rec = recs + ((size_t)head_idx * NCtot + c) * rstride;
                mbar_expect_tx(bar, a_bytes);
                bulk_load(base + SO_WQ, rec + REC_W, 8192, bar);
                bulk_load(base + SO_WQ + 16384, rec + REC_W + 8192, 8192, bar);
                if (write_o) {
                    if (diag) {
                        bulk_load(base + SO_WQ + 8192, rec + REC_QG, 8192, bar);
                        bulk_load(base + SO_WQ + 24576, rec + REC_QG + 8192, 8192, bar);
                    } else {
                        tma_load_4d(base + SO_WQ + 8192, &tm_q, bar, 0, h, c * CH, b);
                        tma_load_4d(base + SO_WQ + 24576, &tm_q, bar, 64, h, c * CH, b);
                    }
                    bulk_load(base + SO_P, rec + REC_P, 16384, bar);
                }
                if (need_vals) {
                    bulk_load(base + SO_TPP, rec + REC_TPP, 16384, bar);
                    tma_load_4d(base + SO_V, &tm_v, bar, 0, h, c * CH, b);
                    tma_load_4d(base + SO_V + 8192, &tm_v, bar, 64, h, c * CH, b);
                }
            };
            auto load_b = [&](int c, int st) {
                const uint32_t bar = full_b0 + 8 * st;
                const uint32_t base = sbase + st * S_STAGE;
                const uint8_t* rec = recs + ((size_t)head_idx * NCtot + c) * rstride;
                mbar_expect_tx(bar, b_bytes);
                bulk_load(base + SO_KT, rec + REC_KT, 16384, bar);
                bulk_load(base + SO_KTLO, rec + REC_KTLO, 16384, bar);
                bulk_load(sbase + S_SC + st * REC_SCB, rec + REC_SC, REC_SCB, bar);
            };
            int last_a = c0 - 1, last_b = c0 - 1;  // last chunk of each part requested
            for (int i = 0; i < min(NC, 2); ++i) {
                load_a(c0 + i, i);
                load_b(c0 + i, i);
                last_a = last_b = c0 + i;
            }
            for (int c = c0; c < c1; ++c) {
                const int lc = c - c0, st = lc & 1;
                // every MMA of chunk c done: part A of its stage can take chunk c + 2
                if (!mbar_wait_bounded(bar_o0 + 8 * st, (lc >> 1) & 1, kWaitNs)) { aborted = true; break; }
                if (c + 2 < c1) {
                    load_a(c + 2, st);
                    last_a = c + 2;
                }
                // o tile staged and every scalar read: store it, then part B
                if (!mbar_wait_bounded(o_free0 + 8 * st, (lc >> 1) & 1, kWaitNs)) { aborted = true; break; }
                if (write_o) {
                    tma_store_4d(&tm_o, sbase + st * S_STAGE + SO_KT, 0, h, c * CH, b);
                    bulk_commit();
                    bulk_wait_read();
                }
                if (c + 2 < c1) {
                    load_b(c + 2, st);
                    last_b = c + 2;
                }
            }
            if (aborted) {
                atomicOr(&ms->abort, 1u);
                // let loads that may still be landing in shared memory finish
                for (int cc = max(c0, last_a - 1); cc <= last_a; ++cc)
                    (void)mbar_wait_bounded(full_a0 + 8 * ((cc - c0) & 1), ((cc - c0) >> 1) & 1, kWaitNs);
                for (int cc = max(c0, last_b - 1); cc <= last_b; ++cc)
                    (void)mbar_wait_bounded(full_b0 + 8 * ((cc - c0) & 1), ((cc - c0) >> 1) & 1, kWaitNs);
            }
            bulk_wait_all();
        }
        __syncwarp();
    } else if (warp == kIssuerWarp) {
        // ================================ MMA issuer ================================
        if (lane == 0) {
            const uint32_t iu = idesc_bf16(128, 64, false, false);
            const uint32_t iuo = idesc_bf16(128, 128, false, false);
            const uint32_t io = idesc_bf16(128, 64, false, false);
            const uint32_t is = idesc_bf16(128, 128, false, true);
            for (int c = c0; c < c1 && !aborted; ++c) {
                const int lc = c - c0, st = lc & 1;
                const uint32_t stg = sbase + st * S_STAGE;
                if (!mbar_wait_bounded(full_a0 + 8 * st, (lc >> 1) & 1, kWaitNs)) { aborted = true; break; }
                // U'^T = V^T T''^T into U's columns (the previous chunk's U was read before its
                // u_ready arrivals, which this thread has waited for): products V x T'' hi, lo
                if (need_vals) {
                    tc_fence_after();
                    const uint32_t iv = idesc_bf16(128, 64, true, false);
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int s = 0; s < 4; ++s)
                            mma_bf16(tmem + TM_U, smem_desc(stg + SO_V + s * 2048, 8192, 1024),
                                     smem_desc(stg + SO_TPP + part * 8192 + s * 32, 16, 1024), iv, (part | s) > 0);
                }
                // [U^T | O1] = S^T [-W^T | Q^T] (N = 128; the record holds -W), accumulated onto U'
                // and onto the zeroed O1 once the previous chunk's O1 and O2 are read.  K steps {0,1,4,5} read
                // the first half of each thread's S columns, {2,3,6,7} the second.  U takes S as its
                // bf16 hi part only: W is itself one bf16 rounding, and the lo part's share is
                // below that (measured: max|err|/rms of o and S_T 3.3e-3 against 2.7e-3 with both
                // parts, over the headline workload and the stress cases); O1 adds S lo x Q^T below.
                // Without outputs the MMAs are U's alone (N = 64).
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (!mbar_wait_bounded(s_ready0 + 8 * half, lc & 1, kWaitNs)) { aborted = true; break; }
                    if (half == 0 && write_o && lc > 0 && !mbar_wait_bounded(o_read, (lc - 1) & 1, kWaitNs)) {
                        aborted = true;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int s = 2 * half + (j & 1) + 4 * (j >> 1);
                        mma_bf16_ts(tmem + TM_U, tmem + TM_SH + 8 * s,
                                    smem_desc(stg + SO_WQ + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                                    write_o ? iuo : iu, need_vals || (half | j) > 0);
                    }
                }
                if (aborted) break;
                mma_commit(bar_u);
                // O1 += S^T lo Q^T
                if (write_o) {
#pragma unroll
                    for (int s = 0; s < 8; ++s)
                        mma_bf16_ts(tmem + TM_O1, tmem + TM_SL + 8 * s,
                                    smem_desc(stg + SO_WQ + 8192 + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024), io, 1);
                }
                // S^T += U^T Ktil (N = 128): K steps {0,2} (first half of each thread's tokens),
                // then {1,3}; products hi x hi, hi x lo, lo x hi
                const uint32_t ua[3] = {TM_UH, TM_UH, TM_UL};
                const uint32_t kb[3] = {stg + SO_KT, stg + SO_KTLO, stg + SO_KT};
                const uint32_t pb[3] = {stg + SO_P, stg + SO_PLO, stg + SO_P};
                if (!mbar_wait_bounded(full_b0 + 8 * st, (lc >> 1) & 1, kWaitNs)) { aborted = true; break; }
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (!mbar_wait_bounded(u_ready0 + 8 * half, lc & 1, kWaitNs)) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int p = 0; p < 3; ++p)
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int s = half + 2 * j;
                            mma_bf16_ts(tmem + TM_S, tmem + ua[p] + 8 * s, smem_desc(kb[p] + s * 2048, 8192, 1024),
                                        is, 1);
                        }
                }
                if (aborted) break;
                mma_commit(bar_s);
                // O2 = U^T P^T
                if (write_o) {
#pragma unroll
                    for (int p = 0; p < 3; ++p)
#pragma unroll
                        for (int s = 0; s < 4; ++s)
                            mma_bf16_ts(tmem + TM_O2, tmem + ua[p] + 8 * s, smem_desc(pb[p] + s * 32, 16, 1024), io,
                                        (p | s) > 0);
                }
                mma_commit(bar_o0 + 8 * st);
            }
            if (aborted) atomicOr(&ms->abort, 1u);
        }
        __syncwarp();
    } else {
        // ================================ epilogue warps ================================
        // Initial state: thread (dv = row, half ch) holds dk in [64 ch, 64 ch + 64).
        {
            const float g0 = NC > 0 ? __expf(ms->gsum[0] + ms->gsum[1]) : 1.f;
#pragma unroll 1
            for (int q2 = 0; q2 < 2; ++q2) {
                const int dk0 = 64 * ch + 32 * q2;
                float x[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    x[e] = S0p ? S0p[(size_t)(dk0 + e) * DV + row] : ((ident && dk0 + e == row) ? 1.f : 0.f);
                if (Sc && NC > 0) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) Sc[((size_t)c0 * DK + dk0 + e) * DV + row] = x[e];
                }
                uint32_t hp[16], lp[16];
                split_pack<32>(x, hp, lp);
                tmem_st16u(tmem + lane_base + TM_SH + 32 * ch + 16 * q2, hp);
                tmem_st16u(tmem + lane_base + TM_SL + 32 * ch + 16 * q2, lp);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] *= diag ? gl0[dk0 + e] : g0;
                tmem_st32(tmem + lane_base + TM_S + 64 * ch + 32 * q2, x);
            }
            if (write_o) {  // O1 starts at zero: the [U | O1] product always accumulates
                float z[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) z[e] = 0.f;
                tmem_st32(tmem + lane_base + TM_O1 + 32 * ch, z);
            }
            epi_signal(s_ready0, tid);
            if (lane == 0) mbar_arrive(s_ready0 + 8);
        }
        for (int c = c0; c < c1; ++c) {
            const int lc = c - c0, st = lc & 1;
            const bool has_next = c + 1 < c1;
            // ---- U epilogue: U (U' - W S, accumulated) to bf16 hi/lo A operands (thread = dv,
            //      tokens 32 ch .. + 32), released in two halves of 16 tokens
            {
                const bool ok = mbar_wait_bounded(bar_u, lc & 1, kWaitNs);
                if (__any_sync(0xffffffffu, !ok)) { aborted = true; break; }
                tc_fence_after();
                float x[32];
                tmem_ld32(tmem + lane_base + TM_U + 32 * ch, x);
                tmem_ld_wait();
                uint8_t* Ut = Utl ? Utl + (size_t)c * 32768 : nullptr;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t hp[8], lp[8];
                    split_pack<16>(x + 16 * half, hp, lp);
                    tmem_st8u(tmem + lane_base + TM_UH + 16 * ch + 8 * half, hp);
                    tmem_st8u(tmem + lane_base + TM_UL + 16 * ch + 8 * half, lp);
                    epi_signal(u_ready0 + 8 * half, tid);  // the first also covers the master rescale
                }
                // tile images for the backward, read back from TMEM while the S product runs: U(c)
                // hi/lo and the chunk's incoming state S_c hi/lo (still the S operand)
                if (Ut) {
                    uint32_t wh[16], wl[16];
                    tmem_ld16u(tmem + lane_base + TM_UH + 16 * ch, wh);
                    tmem_ld16u(tmem + lane_base + TM_UL + 16 * ch, wl);
                    tmem_ld_wait();
                    st_words_sw128_global(Ut, row, 4 * ch, 4, wh);
                    st_words_sw128_global(Ut + 16384, row, 4 * ch, 4, wl);
                }
                if (Stl)
                    st_tmem_row_global(tmem + lane_base + TM_SH + 32 * ch, tmem + lane_base + TM_SL + 32 * ch,
                                       Stl + (size_t)c * 65536 + ch * 16384, 32768, row);
            }
            // ---- state epilogue: S_{c+1} to hi/lo in two halves (releasing U(c+1)), then the
            //      fp32 master pre-scaled by the next gamma_last
            {
                const bool ok = mbar_wait_bounded(bar_s, lc & 1, kWaitNs);
                if (__any_sync(0xffffffffu, !ok)) { aborted = true; break; }
                tc_fence_after();
                if (has_next) {
                    float x0[32], x1[32];
                    tmem_ld32(tmem + lane_base + TM_S + 64 * ch, x0);
                    tmem_ld32(tmem + lane_base + TM_S + 64 * ch + 32, x1);
                    tmem_ld_wait();
                    {
                        uint32_t hp[16], lp[16];
                        split_pack<32>(x0, hp, lp);
                        tmem_st16u(tmem + lane_base + TM_SH + 32 * ch, hp);
                        tmem_st16u(tmem + lane_base + TM_SL + 32 * ch, lp);
                        epi_signal(s_ready0, tid);
                        split_pack<32>(x1, hp, lp);
                        tmem_st16u(tmem + lane_base + TM_SH + 32 * ch + 16, hp);
                        tmem_st16u(tmem + lane_base + TM_SL + 32 * ch + 16, lp);
                        epi_signal(s_ready0 + 8, tid);
                    }
                    if (Sc) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            Sc[((size_t)(c + 1) * DK + 64 * ch + e) * DV + row] = x0[e];
                            Sc[((size_t)(c + 1) * DK + 64 * ch + 32 + e) * DV + row] = x1[e];
                        }
                    }

                    const float* scs = reinterpret_cast<const float*>(sm + S_SC + st * REC_SCB);
                    if (diag) {  // per key channel: this thread holds dk 64 ch .. 64 ch + 63
                        const float4* sc4 = reinterpret_cast<const float4*>(scs + 64 * ch);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float4 a4 = sc4[e], b4 = sc4[8 + e];
                            x0[4 * e] *= a4.x; x0[4 * e + 1] *= a4.y; x0[4 * e + 2] *= a4.z; x0[4 * e + 3] *= a4.w;
                            x1[4 * e] *= b4.x; x1[4 * e + 1] *= b4.y; x1[4 * e + 2] *= b4.z; x1[4 * e + 3] *= b4.w;
                        }
                    } else {
                        const float gN = scs[CH];
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            x0[e] *= gN;
                            x1[e] *= gN;
                        }
                    }
                    tmem_st32(tmem + lane_base + TM_S + 64 * ch, x0);
                    tmem_st32(tmem + lane_base + TM_S + 64 * ch + 32, x1);
                }
            }
            // ---- output epilogue: o = gamma o O1 + O2 staged as [token][dv] over the consumed
            //      Q and W tiles; the loader stores it
            {
                const bool ok = mbar_wait_bounded(bar_o0 + 8 * st, (lc >> 1) & 1, kWaitNs);
                if (__any_sync(0xffffffffu, !ok)) { aborted = true; break; }
                tc_fence_after();
                if (write_o) {
                    const float* gm = reinterpret_cast<const float*>(sm + S_SC + st * REC_SCB);
                    TOut* stage_o = reinterpret_cast<TOut*>(sm + st * S_STAGE + SO_KT);
                    float o1[32], o2[32];
                    tmem_ld32(tmem + lane_base + TM_O1 + 32 * ch, o1);
                    tmem_ld32(tmem + lane_base + TM_O2 + 32 * ch, o2);
                    tmem_ld_wait();
                    {  // O1 back to zero for the next chunk's accumulating [U | O1] product
                        float z[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) z[e] = 0.f;
                        tmem_st32(tmem + lane_base + TM_O1 + 32 * ch, z);
                    }
                    epi_signal(o_read, tid);  // the next chunk's [U | O1] product may start
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int t = 32 * ch + e;
                        stage_o[t * DV + row] = from_f32<TOut>(fmaf(diag ? 1.f : gm[t], o1[e], o2[e]));
                    }
                    fence_proxy_async();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(o_free0 + 8 * st);
            }
        }
        if (aborted && lane == 0) atomicOr(&ms->abort, 1u);
    }

    __syncthreads();
    if (ms->abort) {
        if (tid == 0) atomicOr(&g_split_error, 1u);
    } else if (NC > 0 && warp < kIssuerWarp && STp) {
        tc_fence_after();
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
            const int dk0 = 64 * ch + 32 * q2;
            float x[32];
            tmem_ld32(tmem + lane_base + TM_S + 64 * ch + 32 * q2, x);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) STp[(size_t)(dk0 + e) * DV + row] = x[e];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
    }
    return n;
}

// Segments per head for the state pass: minimise, in units of one state step,
// pass 1 (two CTAs per segment, one CTA per SM) + pass 2 + the fp32 scan (~1 step per segment).
int choose_nseg_split(int BH, int NC) {
    const int sms = sm_count();
    auto waves = [&](long long ctas) { return (ctas + sms - 1) / sms; };
    const long long base = waves(BH) * (long long)NC;
    long long best_cost = base;
    int best = 1;
    for (int ns = 2; ns <= 64 && ns <= NC; ++ns) {
        const long long per = (NC + ns - 1) / ns;
        const long long cost = waves(2LL * BH * ns) * per + waves((long long)BH * ns) * per + ns;
        if (cost < best_cost) {
            best_cost = cost;
            best = ns;
        }
    }
    return (best > 1 && best_cost * 4 < base * 3) ? best : 1;
}

size_t align1k(size_t x) { return (x + 1023) & ~size_t(1023); }

// Two slabs: the state pass holds one SM per head for the whole sequence, so with few heads
// most SMs idle while it runs.  Splitting the chunks into two slabs lets the second slab's
// preparation run on those SMs while the first slab's state pass runs, the second state pass
// starting from the first one's final state.  Cost model in state steps (one chunk of the
// state pass, ~2.5 us here); a wave of preparation CTAs (four per SM for scalar gating, two for
// diagonal gating) takes prep_wave of them (measured: ~21 us and ~27 us per wave).  Returns
// the first slab's chunk count, or 0 for one run.
// The first slab's preparation has the whole GPU: whole waves, and a last partial wave that
// costs 0.45 + 0.55 x its fill (its CTAs share their SMs with fewer others); the second slab's
// runs beside the state pass and spills onto its SMs when it ends, so it is counted fluidly.
// Calibrated on the B=8 T=2048 H=8 forward (a sweep of the split point: optimum at 18 of 32
// chunks, 151.6 us, against 155.6 us at 20 and 164.9 us as one run).
int choose_slab_split(int BH, int NC, bool diag) {
    const int sms = sm_count();
    if (NC < 8 || 2 * BH > sms) return 0;
    const double per_sm = diag ? 2.0 : 4.0, prep_wave = diag ? 10.4 : 8.5;
    auto prep_all = [&](long long items) {
        const long long slots = (long long)per_sm * sms, full = items / slots;
        const double frac = (double)(items - full * slots) / slots;
        return (full + (frac > 0 ? 0.45 + 0.55 * frac : 0.0)) * prep_wave;
    };
    auto prep_beside = [&](double items) { return items / (per_sm * (sms - BH)) * prep_wave; };
    const double base = prep_all((long long)NC * BH) + NC;
    double best = base;
    int nc1 = 0;
    for (int n1 = 2; n1 <= NC - 2; ++n1) {
        const double t = prep_all((long long)n1 * BH) + std::max<double>(n1 + 2, prep_beside((double)(NC - n1) * BH)) +
                         (NC - n1) + 2;
        if (t < best) {
            best = t;
            nc1 = n1;
        }
    }
    return best < 0.95 * base ? nc1 : 0;
}

struct SplitLayout {
    size_t rec_bytes, seg_off, total;
    int nseg, segc;
    int nc1;          // chunks of the first slab (0: one run)
    size_t slab_off;  // [B*H, Dk, Dv] fp32: the state between the slabs
};

SplitLayout split_layout(const FwdArgs& a) {
    SplitLayout L{};
    const int NC = (a.T + CH - 1) / CH;
    const int BH = a.B * a.H;
    L.rec_bytes = align1k((size_t)BH * NC * (a.diag ? REC_BYTES_D : REC_BYTES));
    L.seg_off = L.rec_bytes;
    const int ns = choose_nseg_split(BH, NC);
    if (ns > 1) {
        L.segc = (NC + ns - 1) / ns;
        L.nseg = (NC + L.segc - 1) / L.segc;
        L.total = L.seg_off + (size_t)3 * BH * L.nseg * DK * DV * sizeof(float);
    } else {
        L.nseg = 1;
        L.segc = NC;
        L.total = L.seg_off;
        L.nc1 = choose_slab_split(BH, NC, a.diag);
        if (L.nc1 > 0) {
            L.slab_off = L.total;
            L.total += (size_t)BH * DK * DV * sizeof(float);
        }
    }
    return L;
}

// A stream per device for the second slab's preparation (created once).
cudaError_t slab_stream(cudaStream_t* out) {
    static std::mutex mu;
    static std::unordered_map<int, cudaStream_t> streams;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = streams.find(dev);
    if (it == streams.end()) {
        cudaStream_t s = nullptr;
        if ((e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking)) != cudaSuccess) return e;
        it = streams.emplace(dev, s).first;
    }
    *out = it->second;
    return cudaSuccess;
}

// 4-D map over the [B, T, H, 128] output (fp32 or bf16) for TMA stores of one chunk's rows of
// one (b, h): box = 128 features x 64 tokens, no swizzle.
bool make_out_map(CUtensorMap* m, void* base, int B, int T, int H, bool bf16) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t elt = bf16 ? 2 : 4;
    cuuint64_t dims[4] = {(cuuint64_t)128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {128 * elt, (cuuint64_t)H * 128 * elt, (cuuint64_t)T * H * 128 * elt};
    cuuint32_t box[4] = {128, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <typename TOut>
cudaError_t launch_state(const CUtensorMap& mq, const FwdArgs& a, const uint8_t* recs, dim3 grid, cudaStream_t st) {
    CUtensorMap mo, mv;
    memset(&mo, 0, sizeof(mo));
    if (a.o != nullptr && !make_out_map(&mo, a.o, a.B, a.T, a.H, a.out_bf16)) return cudaErrorInvalidValue;
    if (!make_map(&mv, a.v, a.B, a.T, a.H)) return cudaErrorInvalidValue;  // V for U' = T'' V (required)
    auto kern = a.diag ? chunk_state_kernel<TOut, true> : chunk_state_kernel<TOut, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S_SMEM);
    if (e != cudaSuccess) return e;
    kern<<<grid, ST, S_SMEM, st>>>(mq, mv, mo, a, recs);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_fwd_split_workspace(const FwdArgs& a) {
    if (!(a.bf16 && a.Dk == 128 && a.Dv == 128 && a.T > 0)) return 0;
    return split_layout(a).total;
}

bool chunk_fwd_diag_tc_supported(const FwdArgs& a) {
    return a.diag && a.bf16 && a.Dk == 128 && a.Dv == 128 && a.T > 0 && a.S_chunks == nullptr &&
           a.T_tiles == nullptr && a.S_tiles == nullptr && a.U_tiles == nullptr && !a.rec_extras;
}

namespace {
// Preparation of chunks [cfirst, cfirst + count) of every head.
cudaError_t launch_prep_range(const FwdArgs& a, void* ws, int cfirst, int count, cudaStream_t st) {
    if (a.diag) {
        CUtensorMap mk, mg;
        if (!make_map(&mk, a.k, a.B, a.T, a.H) || !make_out_map(&mg, const_cast<float*>(a.g), a.B, a.T, a.H, false))
            return cudaErrorInvalidValue;
        cudaError_t e =
            cudaFuncSetAttribute(chunk_prep_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PD_SMEM);
        if (e != cudaSuccess) return e;
        chunk_prep_diag_kernel<<<dim3(count, a.B * a.H), PT, PD_SMEM, st>>>(mk, mg, a, static_cast<uint8_t*>(ws), cfirst);
        return cudaGetLastError();
    }
    CUtensorMap mq, mk;
    if (!make_map(&mq, a.q, a.B, a.T, a.H) || !make_map(&mk, a.k, a.B, a.T, a.H)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P_SMEM);
    if (e != cudaSuccess) return e;
    chunk_prep_kernel<<<dim3(count, a.B * a.H), PT, P_SMEM, st>>>(mq, mk, a, static_cast<uint8_t*>(ws), cfirst);
    return cudaGetLastError();
}
// One non-segmented state-pass run over chunks [f.chunk0, f.chunk0 + f.seg_chunks) of every head.
cudaError_t launch_state_run(const FwdArgs& f, void* ws, cudaStream_t st) {
    CUtensorMap mq;
    if (!make_map(&mq, f.q, f.B, f.T, f.H)) return cudaErrorInvalidValue;
    const uint8_t* recs = static_cast<const uint8_t*>(ws);
    const dim3 grid(f.B * f.H, 1);
    return f.out_bf16 ? launch_state<__nv_bfloat16>(mq, f, recs, grid, st) : launch_state<float>(mq, f, recs, grid, st);
}
}  // namespace

cudaError_t launch_chunk_fwd_split_prep(const FwdArgs& a, void* ws, cudaStream_t st) {
    return launch_prep_range(a, ws, 0, (a.T + CH - 1) / CH, st);
}

cudaError_t launch_chunk_fwd_split_state(const FwdArgs& a, void* ws, cudaStream_t st, int stage) {
    CUtensorMap mq;
    if (!make_map(&mq, a.q, a.B, a.T, a.H)) return cudaErrorInvalidValue;
    const SplitLayout L = split_layout(a);
    const int NC = (a.T + CH - 1) / CH;
    const int BH = a.B * a.H;
    uint8_t* recs = static_cast<uint8_t*>(ws);
    auto state = [&](const FwdArgs& f, dim3 grid) {
        return f.out_bf16 ? launch_state<__nv_bfloat16>(mq, f, recs, grid, st)
                          : launch_state<float>(mq, f, recs, grid, st);
    };
    if (L.nseg <= 1) {  // one run: it is the output pass (stages 1 and 2 have nothing to do)
        if (stage == 1 || stage == 2) return cudaSuccess;
        FwdArgs f = a;
        f.nseg = 1;
        f.seg_chunks = NC;
        f.kinds = 1;
        f.chunk0 = 0;
        return state(f, dim3(BH, 1));
    }
    const size_t SZ = (size_t)DK * DV;
    float* MN = reinterpret_cast<float*>(recs + L.seg_off);  // [2, BH, nseg, DK, DV]
    float* Sstart = MN + 2 * (size_t)BH * L.nseg * SZ;        // [BH, nseg, DK, DV]
    FwdArgs p1 = a;
    p1.S0 = nullptr;
    p1.o = nullptr;
    p1.S_T = MN;
    p1.S_chunks = nullptr;
    p1.S_tiles = nullptr;
    p1.U_tiles = nullptr;
    p1.nseg = L.nseg;
    p1.seg_chunks = L.segc;
    p1.kinds = 2;
    p1.chunk0 = 0;
    cudaError_t e = cudaSuccess;
    if (stage == 0 || stage == 1) e = state(p1, dim3(BH * L.nseg, 2));
    if (e != cudaSuccess) return e;
    if (stage == 0 || stage == 2) e = launch_seg_scan(a.S0, MN, Sstart, a.S_T, BH, L.nseg, st);
    if (e != cudaSuccess || stage == 1 || stage == 2) return e;
    FwdArgs p2 = a;
    p2.S0 = Sstart;
    p2.S_T = nullptr;
    p2.nseg = L.nseg;
    p2.seg_chunks = L.segc;
    p2.kinds = 1;
    p2.chunk0 = 0;
    return state(p2, dim3(BH * L.nseg, 1));
}

cudaError_t launch_chunk_fwd_split(const FwdArgs& a, void* ws, cudaStream_t st) {
    const SplitLayout L = split_layout(a);
    if (L.nc1 <= 0) {
        cudaError_t e = launch_chunk_fwd_split_prep(a, ws, st);
        return e == cudaSuccess ? launch_chunk_fwd_split_state(a, ws, st) : e;
    }
    // Two slabs: prep(slab 1) then state(slab 1) on the caller's stream -- the state pass, next
    // in the same queue, takes its SMs (one per head) first -- while prep(slab 2) runs on the
    // side stream over the other SMs; state(slab 2) follows on the caller's stream once both are
    // done.  The kernels of the two streams share no data and never wait on each other.
    const int NC = (a.T + CH - 1) / CH;
    float* Smid = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.slab_off);
    cudaStream_t side = nullptr;
    cudaEvent_t ev_prep = nullptr, ev_state = nullptr;
    cudaError_t e = slab_stream(&side);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_prep, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_state, cudaEventDisableTiming);
    if (e == cudaSuccess) e = launch_prep_range(a, ws, 0, L.nc1, st);
    if (e == cudaSuccess) e = cudaEventRecord(ev_prep, st);
    if (e == cudaSuccess) {
        FwdArgs f1 = a;
        f1.nseg = 1;
        f1.kinds = 1;
        f1.chunk0 = 0;
        f1.seg_chunks = L.nc1;
        f1.S_T = Smid;
        e = launch_state_run(f1, ws, st);
    }
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side, ev_prep, 0);
    if (e == cudaSuccess) {
        e = launch_prep_range(a, ws, L.nc1, NC - L.nc1, side);
        // the caller's stream takes the side stream's work back whatever happens next
        const cudaError_t er = cudaEventRecord(ev_state, side);
        const cudaError_t ej = er == cudaSuccess ? cudaStreamWaitEvent(st, ev_state, 0) : er;
        if (e == cudaSuccess) e = ej;
    }
    if (e == cudaSuccess) {
        FwdArgs f2 = a;
        f2.nseg = 1;
        f2.kinds = 1;
        f2.chunk0 = L.nc1;
        f2.seg_chunks = NC - L.nc1;
        f2.S0 = Smid;
        e = launch_state_run(f2, ws, st);
    }
    if (ev_prep) cudaEventDestroy(ev_prep);  // released once the work that uses them is done
    if (ev_state) cudaEventDestroy(ev_state);
    return e;
}

int chunk_fwd_split_launches(const FwdArgs& a) {
    const SplitLayout L = split_layout(a);
    return L.nseg > 1 ? 4 : (L.nc1 > 0 ? 4 : 2);
}

int chunk_fwd_split_segments(const FwdArgs& a) { return split_layout(a).nseg; }

int reverse_nseg(int BH, int NC) { return choose_nseg_split(BH, NC); }

cudaError_t split_side_stream(cudaStream_t* out) { return slab_stream(out); }

// Two slabs for the backward's reverse pass (one run per head): the reverse pass over the newest
// n1 chunks first, then over the rest while the gradient kernel (one CTA per SM) takes the
// newest chunks on the SMs the reverse pass leaves free; the older chunks' gradient kernel runs
// on every SM at the end.  Cost model in microseconds, calibrated on the B=4 T=4096 H=16
// training backward (reverse pass 228 us over 64 chunks: about 14 us per launch + 3.3 us per
// chunk; gradient kernel 521 us over 4096 items: 18.8 us per wave of one CTA per SM).  Returns
// n1, or 0 for one run.
int bwd_slab_newest(int BH, int NC) {
    const int sms = sm_count();
    if (NC < 8 || 2 * BH > sms) return 0;
    const double F = 14.0, r = 3.3, g = 18.8;
    auto waves = [](long long items, long long slots) { return (double)((items + slots - 1) / slots); };
    const double base = F + r * NC + waves((long long)NC * BH, sms) * g;
    double best = base;
    int n1 = 0;
    for (int k = 2; k <= NC - 2; ++k) {
        const double t = F + r * k + std::max(F + r * (NC - k), waves((long long)k * BH, sms - BH) * g) +
                         waves((long long)(NC - k) * BH, sms) * g;
        if (t < best) {
            best = t;
            n1 = k;
        }
    }
    return best < 0.95 * base ? n1 : 0;
}

cudaError_t split_take_error(cudaStream_t st, unsigned int* flag) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(flag, g_split_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_split_error, &zero, sizeof(unsigned int));
}

}  // namespace kla
