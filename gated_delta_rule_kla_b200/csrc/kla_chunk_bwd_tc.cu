// kla_chunk_bwd_tc.cu -- chunkwise KLA backward on the 5th-generation tensor cores (sm_100a).
//
// Gradients of the split forward (kla_chunk_split.cu; "Kaczmarz Linear Attention", section 4,
// Eqs. 7-9, on unit keys khat = k/r with b = eta r^2/(r^2+eps), c = eta r/(r^2+eps)).  Per
// chunk, with S the incoming state, U = T R the chunk's transformed values (R = Diag(c) V -
// Diag(b gamma) Khat S) and lambda = dS' the gradient of the chunk's outgoing state:
//   dU      = P^T dO + Ktil lambda,       dR = T^T dU
//   dS      = gamma_last lambda + (Diag(gamma) Q)^T dO - W^T dU      (W^T dU = (b gamma Khat)^T dR)
// so the reverse state recurrence needs only the forward's preparation records (P, Ktil, -W)
// and the chunk's dO and Q.  Then, for every chunk independently,
//   Y = dO U^T,  D = -dR U^T,   F = Gam o Y (lower),  E = Diag(b) (Gam^- o D) (strictly lower)
//   dq    = Diag(gamma) dO S^T + F Khat
//   dkhat = -Diag(b gamma) dR S^T + Diag(delta) U lambda^T + F^T Q + (E + E^T) Khat
//   dv    = Diag(c) dR
//   db_i  = sum_t D_it (Gam^- o Khat Khat^T)_it - gamma_i dR_i.(Khat S)_i,   dc_i = dR_i . v_i
//   dG    from every decay factor (Gam, gamma, delta, gamma_last); dg = reverse cumsum of dG
// and dk, deta through the key-norm map of (b, c, khat).
//
// Four steps, all asynchronous on the caller's stream:
//   1. the split forward's preparation kernel (records, plus every chunk's T as bf16 hi/lo)
//   2. the split forward's state pass (every chunk's S and U)
//   3. `chunk_bwd_state_kernel`: one CTA per head walks the chunks backwards carrying lambda in
//      TMEM (warp-specialised like the forward state pass) and stores every chunk's lambda and
//      dR = T^T dU, and dS0
//   4. `chunk_bwd_grad_kernel`: one CTA per (chunk, head); every contraction above on the
//      tensor cores, the masks, decays and per-token scalars on the CUDA cores.
#include <cuda.h>
#include <string.h>

#include "kla_device.cuh"
#include "kla_launch.h"
#include "kla_sm100.cuh"
#include "kla_tc_common.cuh"

namespace kla {

__device__ unsigned int g_bwd_error = 0;

namespace {

using namespace sm100;
using namespace tcc;

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ float ld_sw128_bf16(const uint8_t* blk, int r, int col) {
    const uint32_t off = r * 128 + ((((uint32_t)col >> 3) ^ (uint32_t)(r & 7)) << 4) + (col & 7) * 2;
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(blk + off));
}
// The 16-byte chunk c (8 features) of row r of a 128-byte-swizzled tile.
__device__ __forceinline__ void ld_sw128_chunk(const uint8_t* blk, int r, int c, float* f) {
    unpack_bf16x8(*reinterpret_cast<const uint4*>(blk + r * 128 + ((c ^ (r & 7)) << 4)), f);
}

template <typename TOut>
__device__ __forceinline__ void st_row32(TOut* dst, const float* x);
template <>
__device__ __forceinline__ void st_row32<float>(float* dst, const float* x) {
#pragma unroll
    for (int u = 0; u < 8; ++u)
        reinterpret_cast<float4*>(dst)[u] = make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
}
template <>
__device__ __forceinline__ void st_row32<__nv_bfloat16>(__nv_bfloat16* dst, const float* x) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        uint4 w;
        w.x = pack_bf16x2(x[8 * u], x[8 * u + 1]);
        w.y = pack_bf16x2(x[8 * u + 2], x[8 * u + 3]);
        w.z = pack_bf16x2(x[8 * u + 4], x[8 * u + 5]);
        w.w = pack_bf16x2(x[8 * u + 6], x[8 * u + 7]);
        reinterpret_cast<uint4*>(dst)[u] = w;
    }
}

// Split 8 fp32 values into bf16 hi/lo and store them as 16-byte piece `cc` of row r of two
// 128-byte-swizzled tiles.
__device__ __forceinline__ void st_piece_split(uint8_t* hi_blk, uint8_t* lo_blk, int r, int cc, const float* x) {
    uint4 hh, ll;
    split_chunk8(x, hh, ll);
    const uint32_t off = r * 128 + ((cc ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(hi_blk + off) = hh;
    *reinterpret_cast<uint4*>(lo_blk + off) = ll;
}
template <typename TOut>
__device__ __forceinline__ void st_piece8(TOut* dst, const float* x);
template <>
__device__ __forceinline__ void st_piece8<float>(float* dst, const float* x) {
    reinterpret_cast<float4*>(dst)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
template <>
__device__ __forceinline__ void st_piece8<__nv_bfloat16>(__nv_bfloat16* dst, const float* x) {
    uint4 w;
    w.x = pack_bf16x2(x[0], x[1]);
    w.y = pack_bf16x2(x[2], x[3]);
    w.z = pack_bf16x2(x[4], x[5]);
    w.w = pack_bf16x2(x[6], x[7]);
    *reinterpret_cast<uint4*>(dst) = w;
}

// Device-side view of one backward call: inputs, outputs and the workspace arrays.
struct BwdDev {
    const void *q, *k, *v;
    const float *eta, *g;
    float eps;
    const float* dS_T;
    const uint8_t* recs;   // forward preparation records [BH, NC]
    // per chunk and head, bf16 hi then lo tile images in the 128-byte swizzle:
    const uint8_t* Ttl;    // T: [64 rows of T][64]                                     16 KB
    const uint8_t* Stl;    // incoming state S: [dk half][128 dv rows][64 dk]           64 KB
    const uint8_t* Utl;    // U: [128 dv rows][64 tokens]                               32 KB
    uint8_t* Ltl;          // lambda = dS' (gradient of the outgoing state), as S       64 KB
    float* dR;             // [BH, NC, CH, DV] fp32
    void *dq, *dk, *dv;
    float *deta, *dg, *dS0;
    int B, T, H;
    // Reverse state pass over segments (long sequences over few heads).  mode 0: one run per
    // head from dS_T.  mode 1 (transition pass, grid y = kind): per segment, kind 0 runs from
    // lambda = 0 with dO, kind 1 from lambda = I without dO; the final lambda goes to
    // MN[kind][head][nseg - 1 - seg] (reversed, so that the forward's segment scan chains them
    // newest first).  mode 2 (output pass): per segment from Lstart[head][nseg - 1 - seg] (the
    // scan's output), with the tile and dR stores; dS0 comes from the scan.
    int mode, nseg, segc;
    float* MN;
    const float* Lstart;
    // mode 0 runs chunks [run_lo, run_hi) of every head (from dS_T, the gradient of the state
    // after chunk run_hi - 1, to dS0, that of the state entering chunk run_lo); the gradient
    // kernel takes chunks cfirst + blockIdx.x
    int run_lo, run_hi, cfirst;
};

// =====================================================================================
// Reverse state pass: one CTA per (b, h), chunks newest first.  Warps 0-7 epilogue (thread
// pair = one TMEM lane = one dv column), warp 8 issues the MMAs, warp 9 loads the stages.
// Per chunk (lane = dv throughout; every A operand in TMEM except dO^T):
//   dU^T     = dO^T P + lambda^T Ktil^T          (lambda and Ktil as bf16 hi/lo pairs)
//   lambda^T = gamma_last lambda^T + (gamma dO)^T Q + dU^T (-W)   (master pre-scaled in TMEM)
//   dR^T     = dU^T T
// TMEM: [0,128) lambda^T master fp32, [128,192) lambda^T hi, [192,256) dU^T accumulator,
// [256,288) dU^T hi, [288,320) dU^T lo, [320,352) (gamma dO)^T hi, [352,384) lo,
// [384,448) dR^T accumulator, [448,512) lambda^T lo.  Every chunk's lambda leaves as bf16 hi/lo
// tiles (thread = one dv row of 64 dk: 32-byte stores), the layout the gradient kernel reads.
// =====================================================================================
constexpr int RT = 320;
constexpr int kRIssuer = 8, kRLoader = 9;
constexpr uint32_t R_STAGE = 114688;
constexpr uint32_t SR_DO = 0, SR_Q = 16384, SR_W = 32768, SR_KT = 49152, SR_KTLO = 65536, SR_P = 81920,
                   SR_T = 98304;
static_assert(SR_KT - SR_W == REC_KT - REC_W && SR_KTLO - SR_W == REC_KTLO - REC_W && SR_P - SR_W == REC_P - REC_W &&
                  REC_P + 16384 - REC_W == 65536,
              "the record's -W, Ktil and P tiles arrive as one 64 KB copy");
static_assert(SR_T + 16384 == R_STAGE, "stage size");
constexpr uint32_t R_SC = 2 * R_STAGE;
constexpr uint32_t R_MISC = R_SC + 2 * REC_SCB;
constexpr uint32_t R_SMEM = R_MISC + 128 + 1024;
static_assert(R_SMEM <= 232448, "reverse state pass shared memory");
constexpr uint32_t TR_L = 0, TR_LH = 128, TR_U = 192, TR_UH = 256, TR_UL = 288, TR_GH = 320, TR_GL = 352,
                   TR_R = 384, TR_LL = 448;

struct RevMisc {
    uint64_t full[2], freed[2];
    uint64_t bar_u, bar_s, bar_r;
    uint64_t l_ready[2], u_ready[2], gd_ready;
    uint32_t tmem_base, abort;
    float gsum[2];
};
static_assert(sizeof(RevMisc) <= 128, "reverse pass barriers");

__global__ void __launch_bounds__(RT, 1)
    chunk_bwd_state_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                           BwdDev a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    RevMisc* ms = reinterpret_cast<RevMisc*>(sm + R_MISC);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = tid & 127;      // TMEM lane = dv (epilogue warps)
    const int ch = (tid >> 7) & 1;  // half of every epilogue's columns
    const int H = a.H, T = a.T;
    const int NC = (T + CH - 1) / CH;
    const int nseg = a.mode == 0 ? 1 : a.nseg;
    const int head = blockIdx.x / nseg, seg = blockIdx.x % nseg, b = head / H, h = head % H;
    const int c_lo = a.mode == 0 ? a.run_lo : seg * a.segc, c_hi = a.mode == 0 ? a.run_hi : min(NC, c_lo + a.segc);
    const int nch = c_hi > c_lo ? c_hi - c_lo : 0;  // chunks of this run, processed newest first
    const bool ident = a.mode == 1 && blockIdx.y == 1;  // transition from lambda = I, no dO
    const bool need_do = !ident;
    const bool outputs = a.mode != 1;                   // lambda tiles and dR for the gradient kernel
    const uint32_t sbase = smem_u32(sm);
    const uint32_t full0 = smem_u32(&ms->full[0]), freed0 = smem_u32(&ms->freed[0]);
    const uint32_t bar_u = smem_u32(&ms->bar_u), bar_s = smem_u32(&ms->bar_s), bar_r = smem_u32(&ms->bar_r);
    const uint32_t l_ready0 = smem_u32(&ms->l_ready[0]), u_ready0 = smem_u32(&ms->u_ready[0]),
                   gd_ready = smem_u32(&ms->gd_ready);
    const float* dST = a.mode == 0 ? (a.dS_T ? a.dS_T + (size_t)head * DK * DV : nullptr)
                                   : (a.mode == 2 ? a.Lstart + ((size_t)head * nseg + (nseg - 1 - seg)) * DK * DV
                                                  : nullptr);
    uint8_t* Ltl = a.Ltl + (size_t)head * NC * 65536;
    float* dRh = a.dR + (size_t)head * NC * CH * DV;

    if (tid == 0) {
        mbar_init(full0, 1);
        mbar_init(full0 + 8, 1);
        mbar_init(freed0, 1);
        mbar_init(freed0 + 8, 1);
        mbar_init(bar_u, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_r, 1);
        mbar_init(l_ready0, 8);
        mbar_init(l_ready0 + 8, 8);
        mbar_init(u_ready0, 8);
        mbar_init(u_ready0 + 8, 8);
        mbar_init(gd_ready, 8);
        ms->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ms->tmem_base), 512);
        tmem_relinquish();
    }
    if (warp < 2) {  // gamma_last of the run's newest chunk
        const int t = (c_hi - 1) * CH + tid;
        const float gv = (nch > 0 && t < T) ? a.g[tok_index(b, t, h, T, H)] : 0.f;
        const float sg = warp_sum(gv);
        if (lane == 0) ms->gsum[warp] = sg;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms->tmem_base;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

    bool aborted = false;
    if (warp == kRLoader) {
        // ================================ loader ================================
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_do);
            // without dO (the identity transition) neither dO, Q nor T is needed
            const uint32_t kBytes = 65536 + REC_SCB + (need_do ? 16384 + 4 * 8192 : 0);
            auto load = [&](int c, int st) {
                const uint32_t bar = full0 + 8 * st;
                const uint32_t base = sbase + st * R_STAGE;
                const uint8_t* rec = a.recs + ((size_t)head * NC + c) * REC_BYTES;
                mbar_expect_tx(bar, kBytes);
                bulk_load(base + SR_W, rec + REC_W, 65536, bar);
                bulk_load(sbase + R_SC + st * REC_SCB, rec + REC_SC, REC_SCB, bar);
                if (need_do) {
                    bulk_load(base + SR_T, a.Ttl + ((size_t)head * NC + c) * 16384, 16384, bar);
                    tma_load_4d(base + SR_DO, &tm_do, bar, 0, h, c * CH, b);
                    tma_load_4d(base + SR_DO + 8192, &tm_do, bar, 64, h, c * CH, b);
                    tma_load_4d(base + SR_Q, &tm_q, bar, 0, h, c * CH, b);
                    tma_load_4d(base + SR_Q + 8192, &tm_q, bar, 64, h, c * CH, b);
                }
            };
            int requested = 0;  // chunks (in processing order) whose loads were issued
            for (int i = 0; i < min(nch, 2); ++i) {
                load(c_hi - 1 - i, i);
                requested = i + 1;
            }
            for (int lc = 0; lc + 2 < nch; ++lc) {
                const int st = lc & 1;
                // every MMA of chunk lc done (the epilogue's reads of the stage precede them)
                if (!mbar_wait_bounded(freed0 + 8 * st, (lc >> 1) & 1, kWaitNs)) { aborted = true; break; }
                load(c_hi - 1 - (lc + 2), st);
                requested = lc + 3;
            }
            if (aborted) {
                atomicOr(&ms->abort, 1u);
                // let copies that may still be landing finish (one outstanding phase per stage)
                for (int lc = max(0, requested - 2); lc < requested; ++lc)
                    (void)mbar_wait_bounded(full0 + 8 * (lc & 1), (lc >> 1) & 1, kWaitNs);
            }
        }
        __syncwarp();
    } else if (warp == kRIssuer) {
        // ================================ MMA issuer ================================
        if (lane == 0) {
            const uint32_t i_dop = idesc_bf16(128, 64, true, true);   // dO^T (MN-major) x P (MN-major)
            const uint32_t i_lk = idesc_bf16(128, 64, false, false);  // lambda^T x Ktil^T (K-major)
            const uint32_t i_q = idesc_bf16(128, 128, false, true);   // (gamma dO)^T x Q (MN-major)
            const uint32_t i_w = idesc_bf16(128, 128, false, true);   // dU^T x (-W) ([token][dk] tiles: MN-major)
            const uint32_t i_t = idesc_bf16(128, 64, false, true);    // dU^T x T (MN-major)
            for (int lc = 0; lc < nch && !aborted; ++lc) {
                const int st = lc & 1;
                const uint32_t stg = sbase + st * R_STAGE;
                if (!mbar_wait_bounded(full0 + 8 * st, (lc >> 1) & 1, kWaitNs)) { aborted = true; break; }
                tc_fence_after();
                // dU^T = dO^T P (independent of lambda), then + lambda^T Ktil^T by halves of lambda
                // (products hi x hi, hi x lo, lo x hi): K steps {0,1,4,5} read the first half of
                // each thread's lambda columns.  Without dO the first lambda product starts dU.
                if (need_do) {
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int s = 0; s < 4; ++s)
                            mma_bf16(tmem + TR_U, smem_desc(stg + SR_DO + s * 2048, 8192, 1024),
                                     smem_desc(stg + SR_P + p * 8192 + s * 2048, 8192, 1024), i_dop, (p | s) > 0);
                }
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (!mbar_wait_bounded(l_ready0 + 8 * half, lc & 1, kWaitNs)) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int p = 0; p < 3; ++p)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int s = 2 * half + (j & 1) + 4 * (j >> 1);
                            mma_bf16_ts(tmem + TR_U, tmem + (p == 2 ? TR_LL : TR_LH) + 8 * s,
                                        smem_desc(stg + (p == 1 ? SR_KTLO : SR_KT) + (s >> 2) * 8192 + (s & 3) * 32,
                                                  16, 1024),
                                        i_lk, (need_do || half > 0 || p > 0 || j > 0) ? 1u : 0u);
                        }
                }
                if (aborted) break;
                mma_commit(bar_u);
                // lambda^T += (gamma dO)^T Q, once gamma dO is in TMEM and the master rescaled
                if (need_do) {
                    if (!mbar_wait_bounded(gd_ready, lc & 1, kWaitNs)) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int s = 0; s < 4; ++s)
                            mma_bf16_ts(tmem + TR_L, tmem + (p ? TR_GL : TR_GH) + 8 * s,
                                        smem_desc(stg + SR_Q + s * 2048, 8192, 1024), i_q, 1);
                }
                // lambda^T += dU^T (-W): token steps {0,2} (first half of each thread's tokens),
                // then {1,3}; dU hi and lo against the one-bf16 W
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (!mbar_wait_bounded(u_ready0 + 8 * half, lc & 1, kWaitNs)) { aborted = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int p = 0; p < 2; ++p)
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int s = half + 2 * j;
                            mma_bf16_ts(tmem + TR_L, tmem + (p ? TR_UL : TR_UH) + 8 * s,
                                        smem_desc(stg + SR_W + s * 2048, 8192, 1024), i_w, 1);
                        }
                }
                if (aborted) break;
                mma_commit(bar_s);
                // dR^T = dU^T T: products hi x hi, hi x lo, lo x hi (only for the gradient kernel)
                if (outputs) {
                    const uint32_t ua[3] = {TR_UH, TR_UH, TR_UL};
                    const uint32_t tb[3] = {stg + SR_T, stg + SR_T + 8192, stg + SR_T};
#pragma unroll
                    for (int p = 0; p < 3; ++p)
#pragma unroll
                        for (int s = 0; s < 4; ++s)
                            mma_bf16_ts(tmem + TR_R, tmem + ua[p] + 8 * s, smem_desc(tb[p] + s * 2048, 8192, 1024),
                                        i_t, (p | s) > 0);
                    mma_commit(bar_r);
                }
                mma_commit(freed0 + 8 * st);
            }
            if (aborted) atomicOr(&ms->abort, 1u);
        }
        __syncwarp();
    } else {
        // ================================ epilogue warps ================================
        // lambda of the newest chunk = dS_T (or zero): thread (dv = row, half ch) holds dk in
        // [64 ch, 64 ch + 64); the master is pre-scaled by that chunk's gamma_last.
        {
            const float g0 = __expf(ms->gsum[0] + ms->gsum[1]);
#pragma unroll 1
            for (int q2 = 0; q2 < 2; ++q2) {
                const int dk0 = 64 * ch + 32 * q2;
                float x[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    x[e] = ident ? (dk0 + e == row ? 1.f : 0.f) : (dST ? dST[(size_t)(dk0 + e) * DV + row] : 0.f);
                uint32_t hp[16], lp[16];
                split_pack<32>(x, hp, lp);
                tmem_st16u(tmem + lane_base + TR_LH + 32 * ch + 16 * q2, hp);
                tmem_st16u(tmem + lane_base + TR_LL + 32 * ch + 16 * q2, lp);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] *= g0;
                tmem_st32(tmem + lane_base + TR_L + 64 * ch + 32 * q2, x);
                epi_signal(l_ready0 + 8 * q2, tid);
            }
        }
        // (gamma dO)^T hi/lo for the chunk of processing index lc2 (thread = dv, tokens 32 ch ..
        // + 32), and that chunk's gamma_last of chunk c - 1 for the master's next pre-scale; the
        // signal also orders the master rescale before the Q product
        float gprev = 1.f;
        auto gamma_do = [&](int lc2) -> bool {
            const int st2 = lc2 & 1;
            const bool ok = mbar_wait_bounded(full0 + 8 * st2, (lc2 >> 1) & 1, kWaitNs);
            if (__any_sync(0xffffffffu, !ok)) return false;
            const float* sc = reinterpret_cast<const float*>(sm + R_SC + st2 * REC_SCB);
            gprev = sc[CH + 1];
            if (!need_do) return true;
            const uint8_t* dob = sm + st2 * R_STAGE + SR_DO + (row >> 6) * 8192;
            float x[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int t = 32 * ch + e;
                x[e] = sc[t] * ld_sw128_bf16(dob, t, row & 63);
            }
            uint32_t hp[16], lp[16];
            split_pack<32>(x, hp, lp);
            tmem_st16u(tmem + lane_base + TR_GH + 16 * ch, hp);
            tmem_st16u(tmem + lane_base + TR_GL + 16 * ch, lp);
            epi_signal(gd_ready, tid);
            return true;
        };
        if (nch > 0 && !gamma_do(0)) aborted = true;
        for (int lc = 0; lc < nch && !aborted; ++lc) {
            const int c = c_hi - 1 - lc;
            const bool has_next = lc + 1 < nch;
            // ---- dU epilogue: hi/lo A operands, released in two halves of 16 tokens
            {
                const bool ok = mbar_wait_bounded(bar_u, lc & 1, kWaitNs);
                if (__any_sync(0xffffffffu, !ok)) { aborted = true; break; }
                tc_fence_after();
                float x[32];
                tmem_ld32(tmem + lane_base + TR_U + 32 * ch, x);
                tmem_ld_wait();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t hp[8], lp[8];
                    split_pack<16>(x + 16 * half, hp, lp);
                    tmem_st8u(tmem + lane_base + TR_UH + 16 * ch + 8 * half, hp);
                    tmem_st8u(tmem + lane_base + TR_UL + 16 * ch + 8 * half, lp);
                    epi_signal(u_ready0 + 8 * half, tid);
                }
                // lambda_c (still the dU product's operand) to its tiles while the W product runs
                if (outputs)
                    st_tmem_row_global(tmem + lane_base + TR_LH + 32 * ch, tmem + lane_base + TR_LL + 32 * ch,
                                       Ltl + (size_t)c * 65536 + ch * 16384, 32768, row);
            }
            // ---- lambda epilogue: hi/lo of the next chunk's lambda in two halves, the master
            //      pre-scaled by gamma_last of chunk c - 1, the next chunk's gamma dO
            {
                const bool ok = mbar_wait_bounded(bar_s, lc & 1, kWaitNs);
                if (__any_sync(0xffffffffu, !ok)) { aborted = true; break; }
                tc_fence_after();
                if (has_next) {
                    float x0[32], x1[32];
                    tmem_ld32(tmem + lane_base + TR_L + 64 * ch, x0);
                    tmem_ld32(tmem + lane_base + TR_L + 64 * ch + 32, x1);
                    tmem_ld_wait();
                    {
                        uint32_t hp[16], lp[16];
                        split_pack<32>(x0, hp, lp);
                        tmem_st16u(tmem + lane_base + TR_LH + 32 * ch, hp);
                        tmem_st16u(tmem + lane_base + TR_LL + 32 * ch, lp);
                        epi_signal(l_ready0, tid);
                        split_pack<32>(x1, hp, lp);
                        tmem_st16u(tmem + lane_base + TR_LH + 32 * ch + 16, hp);
                        tmem_st16u(tmem + lane_base + TR_LL + 32 * ch + 16, lp);
                        epi_signal(l_ready0 + 8, tid);
                    }
                    {
                        float y[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) y[e] = x0[e] * gprev;
                        tmem_st32(tmem + lane_base + TR_L + 64 * ch, y);
#pragma unroll
                        for (int e = 0; e < 32; ++e) y[e] = x1[e] * gprev;
                        tmem_st32(tmem + lane_base + TR_L + 64 * ch + 32, y);
                    }
                    if (!gamma_do(lc + 1)) { aborted = true; break; }

                }
            }
            // ---- dR epilogue: dR as [token][dv] rows to the workspace
            if (outputs) {
                const bool ok = mbar_wait_bounded(bar_r, lc & 1, kWaitNs);
                if (__any_sync(0xffffffffu, !ok)) { aborted = true; break; }
                tc_fence_after();
                float x[32];
                tmem_ld32(tmem + lane_base + TR_R + 32 * ch, x);
                tmem_ld_wait();
                float* dr = dRh + (size_t)c * CH * DV;
#pragma unroll
                for (int e = 0; e < 32; ++e) dr[(size_t)(32 * ch + e) * DV + row] = x[e];
                tc_fence_before();
            }
        }
        if (aborted && lane == 0) atomicOr(&ms->abort, 1u);
    }

    __syncthreads();
    if (ms->abort) {
        if (tid == 0) atomicOr(&g_bwd_error, 1u);
    } else if (warp < kRIssuer && a.mode != 2) {
        tc_fence_after();
        // the gradient of the run's oldest state: dS0, or the segment's map in the transition pass
        float* dS0 = a.mode == 0 ? a.dS0 + (size_t)head * DK * DV
                                 : a.MN + (((size_t)blockIdx.y * (gridDim.x / nseg) + head) * nseg + (nseg - 1 - seg)) *
                                              DK * DV;
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
            const int dk0 = 64 * ch + 32 * q2;
            float x[32];
            tmem_ld32(tmem + lane_base + TR_L + 64 * ch + 32 * q2, x);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) dS0[(size_t)(dk0 + e) * DV + row] = x[e];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// =====================================================================================
// Gradient kernel: one CTA (256 threads) per (chunk, head), everything of the chunk in one
// pass.  Shared memory (1024-aligned tiles, 128-byte swizzle, K-major unless noted):
//   [Q; K]        32 KB  kblk k at 16 KB k: rows 0-63 Q, rows 64-127 K (TMA)
//   [dO; dR hi]   32 KB  kblk k at 16 KB k: rows 0-63 dO (TMA), rows 64-127 dR hi
//   dR lo         16 KB  [kblk][64 rows];  U hi, U lo  16 KB each, [kblk][64 rows]
//   S hi/lo       64 KB  [kblk][128 dk rows]; then lambda hi/lo; then the F/E operands
//   F, E fp32     2 x 64 x 65 floats
// The 64-row tiles also serve as the lower half of M = 128 A operands whose upper half is the
// 8 KB before them ("junk" rows whose products land in accumulator lanes that are not read).
// TMEM (512 columns):
//   [0,64)    Gram  [Q; K] K^T          lanes 0-63 Q Khat^T r, 64-127 K K^T (raw keys)
//   [64,128)  [dO; dR_hi] U^T            lanes 0-63 Y, 64-127 dR_hi U^T
//   [128,192) [junk; dR_lo] U_hi^T       lanes 64-127
//   [192,320) [dO; dR_hi] S^T            lanes 0-63 dO S^T, 64-127 dR S^T       (col = dk)
//   [320,448) [junk; U] lambda^T         lanes 64-127 U lambda^T
//   [0,128)   X (after the first two are read): lanes 0-63 F Khat, lanes 64-127
//             (E + E^T) Khat + F^T Q
// =====================================================================================
constexpr int GT = 512;
constexpr uint32_t G_QK = 0, G_DOR = 32768, G_DRL = 65536, G_UH = 81920, G_UL = 98304, G_SL = 114688,
                   G_F = 180224, G_E = G_F + 64 * 65 * 4, G_MISC = G_E + 64 * 65 * 4;
constexpr uint32_t TG_G = 0, TG_YA = 64, TG_YB = 128, TG_Z = 192, TG_L = 320, TG_X = 0;

struct GradMisc {
    uint64_t full, bar1, bar2, bar3, bar_lam;
    uint32_t tmem_base, factored;
    float G[CH], gam[CH], del[CH], ginv[CH], bco[CH], cco[CH], invr[CH], eta[CH], r2[CH], graw[CH];
    // per-token sums over several warps: one slot per contributing warp, added in a fixed order
    float rs_part[8][CH], cs_part[4][CH];
    float rowB_p[4][CH], s_oq_p[4][CH], s_rx_p[4][CH], s_uk_p[4][CH], kd_p[4][CH];
    float kd[CH], dc[CH], dr[CH], dGs[CH];
    float red[GT / 32];
    float lamS;
};
constexpr uint32_t G_SMEM = G_MISC + ((sizeof(GradMisc) + 127) / 128) * 128 + 1024;
static_assert(G_MISC % 8 == 0 && G_SMEM <= 232448, "gradient kernel shared memory");

template <typename TOut>
__global__ void __launch_bounds__(GT, 1)
    chunk_bwd_grad_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_do, BwdDev a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    GradMisc* ms = reinterpret_cast<GradMisc*>(sm + G_MISC);
    float* Fs = reinterpret_cast<float*>(sm + G_F);
    float* Es = reinterpret_cast<float*>(sm + G_E);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, T = a.T;
    const int NC = (T + CH - 1) / CH;
    const int c = a.cfirst + blockIdx.x, head = blockIdx.y;
    const int b = head / H, h = head % H;
    const int t0 = c * CH, n = min(CH, T - t0);
    const size_t crow = (size_t)head * NC + c;  // chunk index in the workspace arrays
    const uint32_t sbase = smem_u32(sm);
    const uint32_t bar_full = smem_u32(&ms->full), bar1 = smem_u32(&ms->bar1), bar2 = smem_u32(&ms->bar2),
                   bar3 = smem_u32(&ms->bar3), bar_lam = smem_u32(&ms->bar_lam);
    // epilogue roles: TMEM lane quadrant and column quarter
    const int q4 = warp & 3, cq = warp >> 2;
    const bool top = q4 < 2;
    const int ti_row = 32 * (q4 & 1) + lane;  // token of this thread's TMEM lane (both halves)
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    uint32_t tmem = 0;
    bool ok = true;
    float dkh[32];  // dkhat of token ti_row, columns [32 cq, 32 cq + 32) (lower-half threads)
    const int pr = tid >> 4, pc = tid & 15;  // 8-feature piece pc of rows pr + 32 j
    const int qq = tid & 3;                   // column quarter when building the F / E operands

    // ---- every input of the chunk requested at once: Q, K, dO by TMA; the S and U tile images
    //      and dR (fp32, into the F/E area) by bulk copies; lambda follows once Z is done
    if (tid == 0) {
        mbar_init(bar_full, 1);
        mbar_init(bar1, 1);
        mbar_init(bar2, 1);
        mbar_init(bar3, 1);
        mbar_init(bar_lam, 1);
        fence_mbar_init();
        mbar_expect_tx(bar_full, 6 * 8192 + 65536 + 32768 + CH * DV * 4);
        tma_load_4d(sbase + G_QK, &tm_q, bar_full, 0, h, t0, b);
        tma_load_4d(sbase + G_QK + 16384, &tm_q, bar_full, 64, h, t0, b);
        tma_load_4d(sbase + G_QK + 8192, &tm_k, bar_full, 0, h, t0, b);
        tma_load_4d(sbase + G_QK + 24576, &tm_k, bar_full, 64, h, t0, b);
        tma_load_4d(sbase + G_DOR, &tm_do, bar_full, 0, h, t0, b);
        tma_load_4d(sbase + G_DOR + 16384, &tm_do, bar_full, 64, h, t0, b);
        bulk_load(sbase + G_SL, a.Stl + crow * 65536, 65536, bar_full);
        bulk_load(sbase + G_UH, a.Utl + crow * 32768, 32768, bar_full);
        bulk_load(sbase + G_F, a.dR + crow * CH * DV, CH * DV * 4, bar_full);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ms->tmem_base), 512);
        tmem_relinquish();
    }
    // Row-major [64][128] arrays are handled in 8-feature pieces: thread tid takes piece pc of
    // rows pr + 32 j (16 consecutive threads share a row).
    uint4 vraw[2];
    {
        uint4 kraw[2];
        float etav[2], gv[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = pr + 32 * j;
            const bool live = i < n;
            const size_t ti = tok_index(b, t0 + (live ? i : 0), h, T, H);
            kraw[j] = live ? reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.k) + ti * DK)[pc]
                           : make_uint4(0u, 0u, 0u, 0u);
            vraw[j] = live ? reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.v) + ti * DV)[pc]
                           : make_uint4(0u, 0u, 0u, 0u);
            etav[j] = live ? a.eta[ti] : 0.f;
            gv[j] = live ? a.g[ti] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = pr + 32 * j;
            float f[8];
            unpack_bf16x8(kraw[j], f);
            float r2 = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) r2 = fmaf(f[e], f[e], r2);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) r2 += __shfl_xor_sync(0xffffffffu, r2, o);
            const KaczCoef cf = kacz_coef(etav[j], r2, a.eps);
            if (pc == 0) {
                ms->graw[i] = gv[j];
                ms->eta[i] = etav[j];
                ms->r2[i] = r2;
                ms->bco[i] = cf.b;
                ms->cco[i] = cf.c;
                ms->invr[i] = cf.inv_r;
            }
        }
    }
    __syncthreads();
    ok = mbar_wait_bounded(bar_full, 0, kWaitNs);
    if (__syncthreads_or(!ok)) goto done;
    // ---- dR: dv = c dR, dc = dR . v, and the dR hi (rows 64-127 of [dO; dR]) / lo tiles
    {
        const float* stg = reinterpret_cast<const float*>(sm + G_F);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = pr + 32 * j;
            const float4 f0 = *reinterpret_cast<const float4*>(stg + i * DV + 8 * pc);
            const float4 f1 = *reinterpret_cast<const float4*>(stg + i * DV + 8 * pc + 4);
            const float x[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
            float vv[8];
            unpack_bf16x8(vraw[j], vv);
            float dcp = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) dcp = fmaf(x[e], vv[e], dcp);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) dcp += __shfl_xor_sync(0xffffffffu, dcp, o);
            if (pc == 0) ms->dc[i] = dcp;
            if (i < n) {
                const float ci = ms->cco[i];
                float y[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) y[e] = ci * x[e];
                st_piece8<TOut>(static_cast<TOut*>(a.dv) + tok_index(b, t0 + i, h, T, H) * DV + 8 * pc, y);
            }
            st_piece_split(sm + G_DOR + (pc >> 3) * 16384 + 8192, sm + G_DRL + (pc >> 3) * 8192, i, pc & 7, x);
        }
    }
    // ---- keys of zero norm.  There the write vanishes and the exact gradient is
    //      dk_t = beta_t Gbar_t v_t (Gbar_t: gradient of the state after token t; Eq. (3) with
    //      ||k_t|| = 0 gives beta_t = eta_t / eps).  The unit-key U holds 0 in column t, and that
    //      column only ever meets khat_t = 0, except in row t of dkhat.  With u_t = beta_t v_t
    //      put in its place, row t of dkhat (F^T Q + E^T Khat + delta_t U lambda^T) is exactly
    //      dk_t, and every other result is unchanged.
    {
        const uint32_t z0 = __ballot_sync(0xffffffffu, lane < n && ms->r2[lane] == 0.f);
        const uint32_t z1 = __ballot_sync(0xffffffffu, lane + 32 < n && ms->r2[lane + 32] == 0.f);
        uint64_t zm = ((uint64_t)z1 << 32) | z0;
        while (zm) {
            const int t = __ffsll((long long)zm) - 1;
            zm &= zm - 1;
            const float bt = a.eps < 0.f ? ms->eta[t] : (a.eps > 0.f ? ms->eta[t] / a.eps : 0.f);
            if (tid < DV && bt != 0.f) {
                const float vt = __bfloat162float(
                    static_cast<const __nv_bfloat16*>(a.v)[tok_index(b, t0 + t, h, T, H) * DV + tid]);
                float hi, lo;
                split_bf16(bt * vt, hi, lo);
                const uint32_t off = tid * 128 + ((((uint32_t)t >> 3) ^ (uint32_t)(tid & 7)) << 4) + (t & 7) * 2;
                *reinterpret_cast<__nv_bfloat16*>(sm + G_UH + off) = __float2bfloat16_rn(hi);
                *reinterpret_cast<__nv_bfloat16*>(sm + G_UL + off) = __float2bfloat16_rn(lo);
            }
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem = ms->tmem_base;
    // ---- MMA group 1: Gram, Y / D, dO S^T and dR S^T (U and S as MN-major B operands)
    if (tid == 0) {
        const uint32_t i64 = idesc_bf16(128, 64, false, false);
        const uint32_t i64n = idesc_bf16(128, 64, false, true);
        const uint32_t i128n = idesc_bf16(128, 128, false, true);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
            mma_bf16(tmem + TG_G, smem_desc(sbase + G_QK + off, 16, 1024), smem_desc(sbase + G_QK + off + 8192, 16, 1024),
                     i64, s > 0);
        }
        // [dO; dR hi] U^T with U hi, then U lo; [junk; dR lo] U hi^T
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16(tmem + TG_YA, smem_desc(sbase + G_DOR + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                         smem_desc(sbase + (p ? G_UL : G_UH) + s * 2048, 8192, 1024), i64n, (p | s) > 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)
            mma_bf16(tmem + TG_YB, smem_desc(sbase + G_DRL - 8192 + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024),
                     smem_desc(sbase + G_UH + s * 2048, 8192, 1024), i64n, s > 0);
        // [dO; dR hi] S^T with S hi, then S lo
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16(tmem + TG_Z, smem_desc(sbase + G_DOR + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                         smem_desc(sbase + G_SL + p * 32768 + s * 2048, 16384, 1024), i128n, (p | s) > 0);
        mma_commit(bar1);
    }
    // ---- meanwhile: the decays (warp 1); this thread's pieces of the S tiles for <lambda, S>
    if (warp == 1) {
        const float x0 = ms->graw[2 * lane], x1 = ms->graw[2 * lane + 1];
        float s = x0 + x1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        const float excl = s - (x0 + x1);
        const float G0 = excl + x0, G1 = excl + x0 + x1;
        ms->G[2 * lane] = G0;
        ms->G[2 * lane + 1] = G1;
        float gr = fmaxf(fabsf(G0), fabsf(G1));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) gr = fmaxf(gr, __shfl_xor_sync(0xffffffffu, gr, o));
        if (lane == 0) ms->factored = gr < 80.f ? 1u : 0u;
    }
    uint4 spc[8];  // hi pieces 0-3 then lo pieces 0-3 (same element positions)
#pragma unroll
    for (int j = 0; j < 8; ++j) spc[j] = reinterpret_cast<const uint4*>(sm + G_SL)[tid + GT * j];
    __syncthreads();
    if (tid < CH) {
        const float Gt = ms->G[tid];
        ms->gam[tid] = __expf(Gt);
        ms->del[tid] = __expf(ms->G[CH - 1] - Gt);  // G is flat past the last token
        ms->ginv[tid] = ms->factored ? __expf(-Gt) : 0.f;
    }
    // ---- lambda tiles over S once group 1 is done (every thread has read its S pieces)
    ok = mbar_wait_bounded(bar1, 0, kWaitNs);
    fence_proxy_async();
    if (__syncthreads_or(!ok)) goto done;
    if (tid == 0) {
        mbar_expect_tx(bar_lam, 65536);
        bulk_load(sbase + G_SL, a.Ltl + crow * 65536, 65536, bar_lam);
    }
    // ---- Gram and Y / D epilogue: F, E to shared memory; row and column sums of the decay
    //      gradient terms (Y o P and D o Diag(b) L), and the L part of db (16 columns a thread)
    {
        const int i = ti_row;
        uint32_t gru[16], yu[16], d2u[16];
        tmem_ld16u(tmem + lane_base + TG_G + 16 * cq, gru);
        tmem_ld16u(tmem + lane_base + TG_YA + 16 * cq, yu);
        if (!top) tmem_ld16u(tmem + lane_base + TG_YB + 16 * cq, d2u);
        tmem_ld_wait();
        const bool fac = ms->factored != 0;
        const float Gi = ms->G[i], gi = ms->gam[i], ir = ms->invr[i], bi = ms->bco[i];
        float rs = 0.f, rb = 0.f, dgv[16];
        if (top) {
            float* Fr = Fs + i * 65;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int t = 16 * cq + e;
                const float y = __uint_as_float(yu[e]);
                const float gm = fac ? gi * ms->ginv[t] : __expf(Gi - ms->G[t]);
                const float gam_it = (t <= i) ? gm : 0.f;
                const float pm = gam_it * __uint_as_float(gru[e]) * ms->invr[t];
                Fr[t] = y * gam_it;
                dgv[e] = y * pm;
                rs += dgv[e];
            }
        } else {
            float* Er = Es + i * 65;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int t = 16 * cq + e;
                const float gm = fac ? gi * ms->ginv[t] : __expf(Gi - ms->G[t]);
                const float gam_it = (t < i) ? gm : 0.f;
                const float D = -(__uint_as_float(yu[e]) + __uint_as_float(d2u[e]));
                const float lh = gam_it * __uint_as_float(gru[e]) * ir * ms->invr[t];
                Er[t] = D * bi * gam_it;
                dgv[e] = D * bi * lh;
                rb = fmaf(D, lh, rb);
                rs += dgv[e];
            }
            ms->rowB_p[cq][i] = rb;
        }
        ms->rs_part[(top ? 0 : 4) + cq][i] = rs;
        // column sums over this warp's 32 rows: lanes 2 m and 2 m + 1 end with column 16 cq + m
#pragma unroll
        for (int off = 16; off >= 2; off >>= 1) {
            const bool up = (lane & off) != 0;
            const int hv = off >> 1;  // values kept after this step
#pragma unroll
            for (int k2 = 0; k2 < hv; ++k2) {
                const float send = up ? dgv[k2] : dgv[k2 + hv];
                const float keep = up ? dgv[k2 + hv] : dgv[k2];
                dgv[k2] = keep + __shfl_xor_sync(0xffffffffu, send, off);
            }
        }
        dgv[0] += __shfl_xor_sync(0xffffffffu, dgv[0], 1);
        if ((lane & 1) == 0) ms->cs_part[q4][16 * cq + (lane >> 1)] = dgv[0];
    }
    // ---- lambda landed: <lambda, S> from the tile pieces, then MMA group 2: [junk; U] lambda^T
    //      (A: U as the upper M half of an MN-major operand, B: lambda MN-major)
    ok = mbar_wait_bounded(bar_lam, 0, kWaitNs);
    if (__syncthreads_or(!ok)) goto done;
    {
        float p = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 lh = reinterpret_cast<const uint4*>(sm + G_SL)[tid + GT * j];
            const uint4 ll = reinterpret_cast<const uint4*>(sm + G_SL)[tid + GT * (j + 4)];
            float a0[8], a1[8], b0[8], b1[8];
            unpack_bf16x8(spc[j], a0);
            unpack_bf16x8(spc[j + 4], a1);
            unpack_bf16x8(lh, b0);
            unpack_bf16x8(ll, b1);
#pragma unroll
            for (int e = 0; e < 8; ++e) p = fmaf(a0[e] + a1[e], b0[e] + b1[e], p);
        }
        p = warp_sum(p);
        if (lane == 0) ms->red[warp] = p;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        const uint32_t i128nn = idesc_bf16(128, 128, true, true);
        const uint32_t ua[3] = {G_UH, G_UH, G_UL};
        const uint32_t lb[3] = {G_SL, G_SL + 32768, G_SL};
#pragma unroll
        for (int p = 0; p < 3; ++p)
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16(tmem + TG_L, smem_desc(sbase + ua[p] - 16384 + s * 2048, 16384, 1024),
                         smem_desc(sbase + lb[p] + s * 2048, 16384, 1024), i128nn, (p | s) > 0);
        mma_commit(bar2);
    } else if (tid == 32) {
        float p = 0.f;
#pragma unroll
        for (int w = 0; w < GT / 32; ++w) p += ms->red[w];
        ms->lamS = p;
    }
    // ---- X operands over the lambda tiles once group 2 is done:
    //      A1 = [F Diag(1/r); (E + E^T) Diag(1/r)],  A2 = [0; F^T]  (hi/lo, 128 rows x 64 tokens)
    ok = mbar_wait_bounded(bar2, 0, kWaitNs);
    if (__syncthreads_or(!ok)) goto done;
    {
        const int r = tid >> 2;  // operand row; this thread's 16 tokens t = 16 qq + e
        float v1[16], v2[16];
        if (r < CH) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int t = 16 * qq + e;
                v1[e] = Fs[r * 65 + t] * ms->invr[t];
                v2[e] = 0.f;
            }
        } else {
            const int i = r - CH;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int t = 16 * qq + e;
                v1[e] = (Es[i * 65 + t] + Es[t * 65 + i]) * ms->invr[t];
                v2[e] = Fs[t * 65 + i];
            }
        }
        st_chunks_split(sm + G_SL, sm + G_SL + 16384, r, 2 * qq, 2, v1);
        st_chunks_split(sm + G_SL + 32768, sm + G_SL + 49152, r, 2 * qq, 2, v2);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        const uint32_t ix = idesc_bf16(128, 128, false, true);
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tmem + TG_X, smem_desc(sbase + G_SL + p * 16384 + s * 32, 16, 1024),
                         smem_desc(sbase + G_QK + (p < 2 ? 8192 : 0) + s * 2048, 16384, 1024), ix, (p | s) > 0);
        mma_commit(bar3);
    }
    ok = mbar_wait_bounded(bar3, 0, kWaitNs);
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    // ---- dq (upper lanes) and dkhat (lower lanes), 32 columns a thread, with their row dot
    //      products (one slot per column quarter)
    {
        const int i = ti_row;
        const bool live = i < n;
        const size_t ti = tok_index(b, t0 + (live ? i : 0), h, T, H);
        const float gi = ms->gam[i];
        if (top) {
            float so = 0.f;
            const uint8_t* qrow = sm + G_QK + (cq >> 1) * 16384;
            float z[32], x[32];
            tmem_ld32(tmem + lane_base + TG_Z + 32 * cq, z);
            tmem_ld32(tmem + lane_base + TG_X + 32 * cq, x);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float f[8];
                ld_sw128_chunk(qrow, i, 4 * (cq & 1) + u, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) so = fmaf(f[e], z[8 * u + e], so);
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = fmaf(gi, z[e], x[e]);
            if (live) st_row32<TOut>(static_cast<TOut*>(a.dq) + ti * DK + 32 * cq, x);
            ms->s_oq_p[cq][i] = so;
        } else {
            float srx = 0.f, suk = 0.f, kdp = 0.f;
            const float nbg = -ms->bco[i] * gi, de = ms->del[i];
            const uint8_t* krow = sm + G_QK + (cq >> 1) * 16384 + 8192;
#pragma unroll
            for (int p = 0; p < 2; ++p) {  // 16 columns at a time (register pressure)
                uint32_t zu[16], lu[16], xu[16];
                tmem_ld16u(tmem + lane_base + TG_Z + 32 * cq + 16 * p, zu);
                tmem_ld16u(tmem + lane_base + TG_L + 32 * cq + 16 * p, lu);
                tmem_ld16u(tmem + lane_base + TG_X + 32 * cq + 16 * p, xu);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    float f[8];
                    ld_sw128_chunk(krow, i, 4 * (cq & 1) + 2 * p + u, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int k2 = 8 * u + e;
                        const float z = __uint_as_float(zu[k2]), l = __uint_as_float(lu[k2]);
                        const float d = fmaf(de, l, fmaf(nbg, z, __uint_as_float(xu[k2])));
                        dkh[16 * p + k2] = d;
                        srx = fmaf(f[e], z, srx);
                        suk = fmaf(f[e], l, suk);
                        kdp = fmaf(f[e], d, kdp);
                    }
                }
            }
            ms->s_rx_p[cq][i] = srx;
            ms->s_uk_p[cq][i] = suk;
            ms->kd_p[cq][i] = kdp;
        }
    }
    __syncthreads();
    // ---- per-token scalars: db, dc -> deta and dr; dG
    if (tid < CH) {
        const int i = tid;
        const float ir = ms->invr[i], gi = ms->gam[i], bi = ms->bco[i], de = ms->del[i];
        auto sum4 = [&](const float (*v)[CH]) { return (v[0][i] + v[1][i]) + (v[2][i] + v[3][i]); };
        const float srx = sum4(ms->s_rx_p) * ir, suk = sum4(ms->s_uk_p) * ir, soq = sum4(ms->s_oq_p);
        const float db = sum4(ms->rowB_p) - gi * srx;
        const float dc = ms->dc[i];
        const float rsum = ((ms->rs_part[0][i] + ms->rs_part[1][i]) + (ms->rs_part[2][i] + ms->rs_part[3][i])) +
                           ((ms->rs_part[4][i] + ms->rs_part[5][i]) + (ms->rs_part[6][i] + ms->rs_part[7][i]));
        const float csum = sum4(ms->cs_part);
        ms->dGs[i] = gi * (soq - bi * srx) - de * suk + rsum - csum;
        float extra = warp_sum(de * suk);  // delta_i = gamma_last / gamma_i feeds dG of the last token
        if (lane == 0) ms->red[warp] = extra;
        const float r2 = ms->r2[i], den = r2 + a.eps, et = ms->eta[i];
        float deta = 0.f, dr = 0.f;
        if (ir > 0.f) {
            const float r = r2 * ir;
            if (a.eps < 0.f) {  // direct: b = eta r^2, c = eta r
                deta = db * r2 + dc * r;
                dr = db * et * 2.f * r + dc * et;
            } else {            // Kaczmarz: b = eta r^2 / (r^2 + eps), c = eta r / (r^2 + eps)
                deta = db * r2 / den + dc * r / den;
                dr = (db * et * 2.f * r * a.eps + dc * et * (a.eps - r2)) / (den * den);
            }
        }
        ms->dr[i] = dr;
        ms->kd[i] = sum4(ms->kd_p) * ir;
        if (i < n) a.deta[tok_index(b, t0 + i, h, T, H)] = deta;
    }
    __syncthreads();
    if (warp == 0) {  // dg = reverse cumulative sum of dG inside the chunk
        float x0 = ms->dGs[2 * lane], x1 = ms->dGs[2 * lane + 1];
        const float add = ms->red[0] + ms->red[1] + ms->gam[n - 1] * ms->lamS;
        if (2 * lane == n - 1) x0 += add;
        if (2 * lane + 1 == n - 1) x1 += add;
        if (2 * lane >= n) x0 = 0.f;
        if (2 * lane + 1 >= n) x1 = 0.f;
        float s = x0 + x1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, s, o);
            if (lane + o < 32) s += y;
        }
        if (2 * lane < n) a.dg[tok_index(b, t0 + 2 * lane, h, T, H)] = s;
        if (2 * lane + 1 < n) a.dg[tok_index(b, t0 + 2 * lane + 1, h, T, H)] = s - x0;
    }
    // ---- dk = (dkhat - khat (khat . dkhat)) / r + khat dr; at a zero-norm key dkhat already
    //      is dk (the substitution in U above)
    if (!top) {
        const int i = ti_row;
        if (i < n) {
            const size_t ti = tok_index(b, t0 + i, h, T, H);
            const float ir = ms->invr[i], kd = ms->kd[i], dr = ms->dr[i];
            const uint8_t* krow = sm + G_QK + (cq >> 1) * 16384 + 8192;
            float x[32];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float f[8];
                ld_sw128_chunk(krow, i, 4 * (cq & 1) + u, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float kh = f[e] * ir;
                    x[8 * u + e] = ir > 0.f ? fmaf(dkh[8 * u + e] - kh * kd, ir, kh * dr) : dkh[8 * u + e];
                }
            }
            st_row32<TOut>(static_cast<TOut*>(a.dk) + ti * DK + 32 * cq, x);
        }
    }
done:
    if (!ok && tid == 0) atomicOr(&g_bwd_error, 2u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(ms->tmem_base, 512);
    }
}

size_t align1k(size_t x) { return (x + 1023) & ~size_t(1023); }

struct BwdLayout {
    size_t fwd, T, S, U, L, dR, seg, mid, total;
    int nseg, segc;
};

// [forward records | T tiles | S tiles | U tiles | lambda tiles | dR | segment maps], each 1 KB
// aligned; the segment maps ([2, BH, nseg] + [BH, nseg] states) only when the reverse state pass
// runs in segments (long sequences over few heads: the forward's cost model)
BwdLayout bwd_layout(int B, int T, int H) {
    FwdArgs fa{};
    fa.B = B;
    fa.T = T;
    fa.H = H;
    fa.Dk = fa.Dv = 128;
    fa.bf16 = true;
    const size_t nch = (size_t)B * H * ((T + CH - 1) / CH);
    BwdLayout L{};
    size_t o = align1k(chunk_fwd_split_workspace(fa));
    L.fwd = 0;
    L.T = o;
    o += align1k(nch * 16384);
    L.S = o;
    o += align1k(nch * 65536);
    L.U = o;
    o += align1k(nch * 32768);
    L.L = o;
    o += align1k(nch * 65536);
    L.dR = o;
    o += align1k(nch * CH * DV * sizeof(float));
    L.seg = o;
    const int NC = (T + CH - 1) / CH;
    const int ns = reverse_nseg(B * H, NC);
    L.nseg = 1;
    L.segc = NC;
    if (ns > 1) {
        L.segc = (NC + ns - 1) / ns;
        L.nseg = (NC + L.segc - 1) / L.segc;
        o += align1k((size_t)3 * B * H * L.nseg * DK * DV * sizeof(float));
    }
    L.mid = o;  // [B*H, DK, DV] fp32: lambda between the two slabs of the reverse pass
    o += align1k((size_t)B * H * DK * DV * sizeof(float));
    L.total = o;
    return L;
}

// The gradient kernel over chunks [cfirst, cfirst + count) of every head.
template <typename TOut>
cudaError_t launch_grad(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mdo, BwdDev d,
                        int cfirst, int count, int BH, cudaStream_t st) {
    if (count <= 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(chunk_bwd_grad_kernel<TOut>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)G_SMEM);
    if (e != cudaSuccess) return e;
    d.cfirst = cfirst;
    chunk_bwd_grad_kernel<TOut><<<dim3(count, BH), GT, G_SMEM, st>>>(mq, mk, mdo, d);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_bwd_tc_workspace(int B, int T, int H, bool have_S_chunks) {
    (void)have_S_chunks;  // the tensor-core path recomputes the states as tiles in any case
    if (B < 1 || H < 1 || T < 1) return 0;
    return bwd_layout(B, T, H).total;
}

cudaError_t launch_chunk_fwd_train_tc(const FwdArgs& f, void* ws, size_t ws_bytes, cudaStream_t st) {
    const BwdLayout L = bwd_layout(f.B, f.T, f.H);
    if (ws == nullptr || ws_bytes < L.total) return cudaErrorInvalidValue;
    uint8_t* w = static_cast<uint8_t*>(ws);
    FwdArgs fa = f;
    fa.T_tiles = w + L.T;
    fa.S_tiles = w + L.S;
    fa.U_tiles = w + L.U;
    return launch_chunk_fwd_split(fa, w + L.fwd, st);  // two slabs when the heads are few
}

cudaError_t launch_chunk_bwd_tc_reverse(const BwdTcArgs& a, void* ws, size_t ws_bytes, cudaStream_t st) {
    const BwdLayout L = bwd_layout(a.B, a.T, a.H);
    if (ws == nullptr || ws_bytes < L.total) return cudaErrorInvalidValue;
    uint8_t* w = static_cast<uint8_t*>(ws);
    CUtensorMap mq, mk, mdo;
    if (!make_map(&mq, a.q, a.B, a.T, a.H) || !make_map(&mk, a.k, a.B, a.T, a.H) ||
        !make_map(&mdo, a.dO, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    BwdDev d{};
    d.q = a.q;
    d.k = a.k;
    d.v = a.v;
    d.eta = a.eta;
    d.g = a.g;
    d.eps = a.eps;
    d.dS_T = a.dS_T;
    d.recs = w + L.fwd;
    d.Ttl = w + L.T;
    d.Stl = w + L.S;
    d.Utl = w + L.U;
    d.Ltl = w + L.L;
    d.dR = reinterpret_cast<float*>(w + L.dR);
    d.dq = a.dq;
    d.dk = a.dk;
    d.dv = a.dv;
    d.deta = a.deta;
    d.dg = a.dg;
    d.dS0 = a.dS0;
    d.B = a.B;
    d.T = a.T;
    d.H = a.H;
    const int BH = a.B * a.H, NC = (a.T + CH - 1) / CH;
    cudaError_t e =
        cudaFuncSetAttribute(chunk_bwd_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)R_SMEM);
    if (e != cudaSuccess) return e;
    auto grad = [&](const BwdDev& dd, int cfirst, int count, cudaStream_t s) {
        return a.out_bf16 ? launch_grad<__nv_bfloat16>(mq, mk, mdo, dd, cfirst, count, BH, s)
                          : launch_grad<float>(mq, mk, mdo, dd, cfirst, count, BH, s);
    };
    if (L.nseg <= 1) {
        d.mode = 0;
        const int n1 = bwd_slab_newest(BH, NC);
        if (n1 <= 0) {
            d.run_lo = 0;
            d.run_hi = NC;
            chunk_bwd_state_kernel<<<BH, RT, R_SMEM, st>>>(mq, mdo, d);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            return grad(d, 0, NC, st);
        }
        // Two slabs: the reverse pass over the newest n1 chunks, then over the rest from the
        // lambda it leaves, on `st` (it takes its SMs, one per head, before the gradient kernel
        // queued beside it); the gradient kernel of the newest chunks runs on the side stream
        // over the other SMs meanwhile, that of the older chunks on `st` once the reverse pass
        // is done, and `st` takes the side stream's work back.  No kernel waits on another.
        const int csplit = NC - n1;
        float* Lmid = reinterpret_cast<float*>(w + L.mid);
        cudaStream_t side = nullptr;
        cudaEvent_t ev_rev = nullptr, ev_grad = nullptr;
        e = split_side_stream(&side);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_rev, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_grad, cudaEventDisableTiming);
        if (e == cudaSuccess) {
            BwdDev d1 = d;
            d1.run_lo = csplit;
            d1.run_hi = NC;
            d1.dS0 = Lmid;
            chunk_bwd_state_kernel<<<BH, RT, R_SMEM, st>>>(mq, mdo, d1);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) e = cudaEventRecord(ev_rev, st);
        if (e == cudaSuccess) {
            BwdDev d2 = d;
            d2.run_lo = 0;
            d2.run_hi = csplit;
            d2.dS_T = Lmid;
            chunk_bwd_state_kernel<<<BH, RT, R_SMEM, st>>>(mq, mdo, d2);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side, ev_rev, 0);
        if (e == cudaSuccess) {
            e = grad(d, csplit, n1, side);
            // the caller's stream takes the side stream's work back whatever happens next
            const cudaError_t er = cudaEventRecord(ev_grad, side);
            if (e == cudaSuccess) e = grad(d, 0, csplit, st);
            const cudaError_t ej = er == cudaSuccess ? cudaStreamWaitEvent(st, ev_grad, 0) : er;
            if (e == cudaSuccess) e = ej;
        }
        if (ev_rev) cudaEventDestroy(ev_rev);  // released once the work that uses them is done
        if (ev_grad) cudaEventDestroy(ev_grad);
        return e;
    } else {
        // transition pass (each segment's map from lambda = I and its offset from lambda = 0),
        // the scan newest segment first (dS_T in, every segment's lambda_end and dS0 out), then
        // each segment's pass from its lambda_end with the tile stores
        const size_t SZ = (size_t)DK * DV;
        float* MN = reinterpret_cast<float*>(w + L.seg);  // [2, BH, nseg, DK, DV]
        float* Lst = MN + 2 * (size_t)BH * L.nseg * SZ;    // [BH, nseg, DK, DV]
        d.nseg = L.nseg;
        d.segc = L.segc;
        d.MN = MN;
        d.Lstart = Lst;
        d.mode = 1;
        chunk_bwd_state_kernel<<<dim3(BH * L.nseg, 2), RT, R_SMEM, st>>>(mq, mdo, d);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if ((e = launch_seg_scan(a.dS_T, MN, Lst, a.dS0, BH, L.nseg, st)) != cudaSuccess) return e;
        d.mode = 2;
        chunk_bwd_state_kernel<<<dim3(BH * L.nseg, 1), RT, R_SMEM, st>>>(mq, mdo, d);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return grad(d, 0, NC, st);
}

cudaError_t launch_chunk_bwd_tc(const BwdTcArgs& a, void* ws, size_t ws_bytes, cudaStream_t st) {
    // 1-2: the forward's records and the T, S and U tiles (no o, S_T or fp32 states)
    FwdArgs fa{};
    fa.q = a.q;
    fa.k = a.k;
    fa.v = a.v;
    fa.eta = a.eta;
    fa.g = a.g;
    fa.eps = a.eps;
    fa.S0 = a.S0;
    fa.B = a.B;
    fa.T = a.T;
    fa.H = a.H;
    fa.Dk = fa.Dv = 128;
    fa.bf16 = true;
    cudaError_t e = launch_chunk_fwd_train_tc(fa, ws, ws_bytes, st);
    // 3-4: reverse state pass and gradients
    return e == cudaSuccess ? launch_chunk_bwd_tc_reverse(a, ws, ws_bytes, st) : e;
}

cudaError_t bwd_tc_take_error(cudaStream_t st, unsigned int* flag) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(flag, g_bwd_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_bwd_error, &zero, sizeof(unsigned int));
}

}  // namespace kla
