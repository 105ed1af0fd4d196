// kla_decode.cu -- single-token KLA decode step ("Kaczmarz Linear Attention", Algorithm 1,
// left panel, lines 2-6), fp32 state updated in place.
//
// Each column j of S evolves on its own given (k, q, alpha, beta):
//   e_j  = v_j - alpha (S^T k)_j
//   S'_ij = alpha S_ij + beta k_i e_j
//   o_j  = (S'^T q)_j = alpha (S^T q)_j + beta (k.q) e_j
// so one pass that reads S once yields both reductions; the update is applied to values
// already on chip and written back once.  The kernel is HBM bound: 2 * Dk * Dv * 4 bytes of
// state traffic per head against ~7 Dk Dv FLOPs.
//
// Work unit = one head's state restricted to NV = 64 value columns (the columns are
// independent): Dk x 64 fp32.  A persistent grid with two CTAs per SM walks the units; a
// single thread keeps up to STAGES - 1 units ahead in flight with 2-D TMA loads (plus 1-D
// bulk copies of k, q and the unit's slice of v) into a ring of shared-memory stages, while
// all threads reduce and update the current unit; the updated tile goes back into its stage
// and leaves by one 2-D TMA store once every warp has written its rows (an mbarrier, so no
// warp waits for the store).  One block-wide barrier per unit: every lane finishes the
// reductions for its own column group from per-warp partials kept in two buffers (by unit
// parity).  Waits are bounded; on expiry the kernel records an error word (reported by
// kla_check_device_error) and stops.
#include <cuda.h>

#include "kla_device.cuh"
#include "kla_launch.h"
#include "kla_sm100.cuh"

namespace kla {

__device__ unsigned int g_decode_error = 0;

namespace {

using namespace sm100;

constexpr int NT = 256;
#ifndef KLA_DECODE_NV
#define KLA_DECODE_NV 64
#endif
#ifndef KLA_DECODE_STAGES
#define KLA_DECODE_STAGES 3
#endif
#ifndef KLA_DECODE_CTAS
#define KLA_DECODE_CTAS 2
#endif
constexpr int NV = KLA_DECODE_NV;         // value columns per unit
constexpr int CG = NV / 4;                // float4 column groups per unit
constexpr int RG = NT / CG;               // row groups
constexpr int STAGES = KLA_DECODE_STAGES;
constexpr int CTAS_PER_SM = KLA_DECODE_CTAS;
static_assert(CG <= 32 && 32 % CG == 0, "column groups tile a warp");
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kInjectedWaitNs = 20000000ull;  // 20 ms: the injected wait (below)

constexpr int NW = NT / 32;       // warps

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
constexpr int MAX_UNITS_PER_CTA = 64;

template <int DK, typename Tin>
struct DecodeSmem {
    float s[STAGES][DK][NV];                    // state tiles
    float gv[STAGES][DK];                       // diagonal gating: the head's per-channel log-decay
    Tin kv[STAGES][DK], qv[STAGES][DK], vv[STAGES][NV];
    float4 red_k[2][NW][CG], red_q[2][NW][CG];  // per-warp partial S^T k, S^T q (by unit parity)
    float scal[2][2][NW];                       // per-warp partial ||k||^2, k.q (by unit parity)
    float alpha[MAX_UNITS_PER_CTA], eta[MAX_UNITS_PER_CTA];
    uint64_t full[STAGES], done[STAGES];        // tile landed; every warp wrote its updated rows
    uint64_t never;                             // failure injection: a barrier nothing completes
};

// DIAG: diagonal gating ("Kaczmarz Linear Attention", App. A.5): g is [B, H, Dk] and row i of
// the state decays by alpha_i = exp(g_i), so alpha_i folds into k_i and q_i in the reductions
// (S-bar^T k = S^T (alpha o k)) and into the update of row i.
template <int DK, int DV, typename Tin, typename TOut, bool DIAG>
__global__ void __launch_bounds__(NT, CTAS_PER_SM)
    decode_step_kernel(const __grid_constant__ CUtensorMap tm_s, const Tin* __restrict__ q,
                       const Tin* __restrict__ k, const Tin* __restrict__ v, const float* __restrict__ eta,
                       const float* __restrict__ g, float eps, float* __restrict__ S, TOut* __restrict__ o,
                       int units, int inject_timeout) {
    constexpr int RPT = DK / RG;   // rows per thread
    constexpr int UPH = DV / NV;   // units per head
    constexpr uint32_t kTileBytes = DK * NV * 4;
    constexpr uint32_t kVecBytes = DK * sizeof(Tin);
    constexpr uint32_t kVBytes = NV * sizeof(Tin);
    extern __shared__ uint8_t smem_raw[];
    auto& sm = *reinterpret_cast<DecodeSmem<DK, Tin>*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cg = tid % CG;
    const int rg = tid / CG;
    const int stride = gridDim.x;
    const int nmine = (blockIdx.x < units) ? (units - 1 - blockIdx.x) / stride + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.done[s]), NW);
        }
        mbar_init(smem_u32(&sm.never), 1);
        fence_mbar_init();
        prefetch_tmap(&tm_s);
    }
    // Launched with programmatic stream serialization: the set-up above touches only shared
    // memory, so it may overlap the previous kernel's tail; the state, inputs and gates it
    // produced are read only after this wait.  The next step may then be scheduled (it waits in
    // the same way for this one to finish).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // one thread requests unit number i of this CTA into stage i % STAGES
    auto request = [&](int i) {
        const int u = blockIdx.x + i * stride;
        const int head = u / UPH, v0 = (u % UPH) * NV;
        const int st = i % STAGES;
        const uint32_t bar = smem_u32(&sm.full[st]);
        mbar_expect_tx(bar, kTileBytes + 2 * kVecBytes + kVBytes + (DIAG ? DK * 4 : 0));
        tma_load_2d(smem_u32(&sm.s[st][0][0]), &tm_s, bar, v0, head * DK);
        if (DIAG) bulk_load(smem_u32(&sm.gv[st][0]), g + (size_t)head * DK, DK * 4, bar);
        bulk_load(smem_u32(&sm.kv[st][0]), k + (size_t)head * DK, kVecBytes, bar);
        bulk_load(smem_u32(&sm.qv[st][0]), q + (size_t)head * DK, kVecBytes, bar);
        bulk_load(smem_u32(&sm.vv[st][0]), v + (size_t)head * DV + v0, kVBytes, bar);
    };
    if (tid == 0) {  // the first tiles are requested before anything else
        for (int i = 0; i < STAGES - 1 && i < nmine; ++i) request(i);
    }
    // the decay and gate of every unit this CTA will process, loaded once
    if (tid < nmine) {
        const int head = (blockIdx.x + tid * stride) / UPH;
        sm.alpha[tid] = DIAG ? 1.f : expf(g[head]);
        sm.eta[tid] = eta[head];
    }
    __syncthreads();


    bool store_failed = false;  // tid 0: a store barrier expired (the next unit's check stops all)
    for (int i = 0; i < nmine; ++i) {
        const int u = blockIdx.x + i * stride;
        const int head = u / UPH, v0 = (u % UPH) * NV;
        const int st = i % STAGES, par = i & 1;
        // keep STAGES - 1 units in flight; the stage refilled now held unit i - 1, whose store
        // was issued at the end of the previous iteration: let it finish reading first
        if (tid == 0 && i + STAGES - 1 < nmine) {
            bulk_wait_read();
            request(i + STAGES - 1);
        }
        bool ok = mbar_wait_bounded(smem_u32(&sm.full[st]), (i / STAGES) & 1, kWaitLimitNs) && !store_failed;
        // failure injection (kla_debug_inject_wait_timeout): the first unit also waits on a
        // barrier that no thread and no copy completes, so that bounded wait expires and the
        // error path below runs exactly as for a lost copy
        if (inject_timeout && i == 0) ok = mbar_wait_bounded(smem_u32(&sm.never), 0, kInjectedWaitNs) && ok;
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(&g_decode_error, 1u);
                // let the loads already requested land before the CTA exits
                const int last = min(i + STAGES - 1, nmine - 1);
                for (int j = i; j <= last; ++j)
                    (void)mbar_wait_bounded(smem_u32(&sm.full[j % STAGES]), (j / STAGES) & 1, kWaitLimitNs);
            }
            break;
        }
        // partial ||k||^2, k.q, S^T k, S^T q; the state slice stays in registers
        float kk = 0.f, kq = 0.f;
        if (tid < DK) {
            const float kx = to_f32(sm.kv[st][tid]), qx = to_f32(sm.qv[st][tid]);
            kk = kx * kx;
            kq = kx * qx;
        }
        float4 cur[RPT];
        float kir[RPT], air[RPT];
        float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int row = rg + r * RG;
            cur[r] = *reinterpret_cast<const float4*>(&sm.s[st][row][4 * cg]);
            air[r] = DIAG ? expf(sm.gv[st][row]) : 1.f;
            kir[r] = to_f32(sm.kv[st][row]);
            const float ki = DIAG ? air[r] * kir[r] : kir[r];
            const float qi = DIAG ? air[r] * to_f32(sm.qv[st][row]) : to_f32(sm.qv[st][row]);
            pk.x = fmaf(cur[r].x, ki, pk.x); pk.y = fmaf(cur[r].y, ki, pk.y);
            pk.z = fmaf(cur[r].z, ki, pk.z); pk.w = fmaf(cur[r].w, ki, pk.w);
            pq.x = fmaf(cur[r].x, qi, pq.x); pq.y = fmaf(cur[r].y, qi, pq.y);
            pq.z = fmaf(cur[r].z, qi, pq.z); pq.w = fmaf(cur[r].w, qi, pq.w);
        }
        // lanes c, c + CG, ... hold the same columns (several rows of the warp): fold them
#pragma unroll
        for (int sh = CG; sh < 32; sh <<= 1) {
            pk.x += __shfl_xor_sync(0xffffffffu, pk.x, sh); pk.y += __shfl_xor_sync(0xffffffffu, pk.y, sh);
            pk.z += __shfl_xor_sync(0xffffffffu, pk.z, sh); pk.w += __shfl_xor_sync(0xffffffffu, pk.w, sh);
            pq.x += __shfl_xor_sync(0xffffffffu, pq.x, sh); pq.y += __shfl_xor_sync(0xffffffffu, pq.y, sh);
            pq.z += __shfl_xor_sync(0xffffffffu, pq.z, sh); pq.w += __shfl_xor_sync(0xffffffffu, pq.w, sh);
        }
        kk = warp_sum(kk);
        kq = warp_sum(kq);
        if (lane < CG) {
            sm.red_k[par][warp][lane] = pk;
            sm.red_q[par][warp][lane] = pq;
        }
        if (lane == 0) {
            sm.scal[par][0][warp] = kk;
            sm.scal[par][1][warp] = kq;
        }
        __syncthreads();
        // every lane: final sums, residual and beta e for its column group cg (== lane % 16)
        const float alpha = sm.alpha[i];
        float4 be;
        {
            float n2 = 0.f, kdq = 0.f;
            float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sq = sk;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                n2 += sm.scal[par][0][w];
                kdq += sm.scal[par][1][w];
                const float4 a = sm.red_k[par][w][cg], b = sm.red_q[par][w][cg];
                sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
                sq.x += b.x; sq.y += b.y; sq.z += b.z; sq.w += b.w;
            }
            const float den = n2 + eps;  // eps < 0: the direct write strength beta = eta
            const float beta = eps < 0.f ? sm.eta[i] : (den > 0.f ? sm.eta[i] / den : 0.f);
            be.x = beta * (to_f32(sm.vv[st][4 * cg + 0]) - alpha * sk.x);
            be.y = beta * (to_f32(sm.vv[st][4 * cg + 1]) - alpha * sk.y);
            be.z = beta * (to_f32(sm.vv[st][4 * cg + 2]) - alpha * sk.z);
            be.w = beta * (to_f32(sm.vv[st][4 * cg + 3]) - alpha * sk.w);
            if (o != nullptr && tid < CG) {  // o = alpha S^T q + (k.q) beta e
                TOut* oh = o + (size_t)head * DV + v0 + tid * 4;
                oh[0] = from_f32<TOut>(fmaf(alpha, sq.x, kdq * be.x));
                oh[1] = from_f32<TOut>(fmaf(alpha, sq.y, kdq * be.y));
                oh[2] = from_f32<TOut>(fmaf(alpha, sq.z, kdq * be.z));
                oh[3] = from_f32<TOut>(fmaf(alpha, sq.w, kdq * be.w));
            }
        }
        // S <- alpha S + beta k e^T into the stage, then out by one TMA store of the tile
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int row = rg + r * RG;
            const float ki = kir[r];
            const float ar = DIAG ? air[r] : alpha;
            float4 x = cur[r];
            x.x = fmaf(ar, x.x, ki * be.x);
            x.y = fmaf(ar, x.y, ki * be.y);
            x.z = fmaf(ar, x.z, ki * be.z);
            x.w = fmaf(ar, x.w, ki * be.w);
            *reinterpret_cast<float4*>(&sm.s[st][row][4 * cg]) = x;
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.done[st]));
        if (tid == 0) {
            if (!mbar_wait_bounded(smem_u32(&sm.done[st]), (i / STAGES) & 1, kWaitLimitNs)) {
                atomicOr(&g_decode_error, 1u);
                store_failed = true;
            } else {
                tma_store_2d(&tm_s, smem_u32(&sm.s[st][0][0]), v0, head * DK);
                bulk_commit();
            }
        }
    }
    if (tid == 0) bulk_wait_all();  // every state tile has left shared memory and reached global
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

template <int DK, int DV, typename Tin, typename TOut, bool DIAG>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t st) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    // the state as a 2-D fp32 matrix [B*H*Dk rows, Dv columns]; box = Dk rows x 64 columns
    CUtensorMap ms;
    cuuint64_t dims[2] = {(cuuint64_t)DV, (cuuint64_t)a.B * a.H * DK};
    cuuint64_t strides[1] = {(cuuint64_t)DV * 4};
    cuuint32_t box[2] = {NV, DK};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&ms, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a.S, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const int units = a.B * a.H * (DV / NV);
    int grid = units < CTAS_PER_SM * sm_count() ? units : CTAS_PER_SM * sm_count();
    if ((units + grid - 1) / grid > MAX_UNITS_PER_CTA) grid = (units + MAX_UNITS_PER_CTA - 1) / MAX_UNITS_PER_CTA;
    const size_t smem = sizeof(DecodeSmem<DK, Tin>) + 128;
    cudaError_t e = cudaFuncSetAttribute(decode_step_kernel<DK, DV, Tin, TOut, DIAG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the previous kernel's tail
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_step_kernel<DK, DV, Tin, TOut, DIAG>, ms, static_cast<const Tin*>(a.q),
                              static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v), a.eta, a.g, a.eps, a.S,
                              static_cast<TOut*>(a.o), units, a.inject_timeout ? 1 : 0);
}

template <int DK, int DV, typename Tin>
cudaError_t launch_decode_o(const DecodeArgs& a, cudaStream_t st) {
    if (a.diag)
        return a.out_bf16 ? launch_decode_t<DK, DV, Tin, __nv_bfloat16, true>(a, st)
                          : launch_decode_t<DK, DV, Tin, float, true>(a, st);
    return a.out_bf16 ? launch_decode_t<DK, DV, Tin, __nv_bfloat16, false>(a, st)
                      : launch_decode_t<DK, DV, Tin, float, false>(a, st);
}

template <typename Tin>
cudaError_t launch_decode_d(const DecodeArgs& a, cudaStream_t st) {
    if (a.Dk == 128 && a.Dv == 128) return launch_decode_o<128, 128, Tin>(a, st);
    if (a.Dk == 128 && a.Dv == 64) return launch_decode_o<128, 64, Tin>(a, st);
    if (a.Dk == 64 && a.Dv == 128) return launch_decode_o<64, 128, Tin>(a, st);
    return launch_decode_o<64, 64, Tin>(a, st);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
    if (a.bf16) return launch_decode_d<__nv_bfloat16>(a, st);
    return launch_decode_d<float>(a, st);
}

cudaError_t decode_take_error(cudaStream_t st, unsigned int* flag) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(flag, g_decode_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(unsigned int));
}

}  // namespace kla
