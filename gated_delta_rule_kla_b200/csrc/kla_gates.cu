// kla_gates.cu -- the gate prologue: the per-token inputs of the KLA recurrence that come from
// the layer's token vector x_t ("Kaczmarz Linear Attention", section 3.3: eta_t is a
// sigmoid-activated linear projection of the input token; alpha_t = exp(g_t)):
//   z_t   = W x_t + bias                    W [2H, D]: rows 0..H-1 eta, rows H..2H-1 decay
//   eta_t = sigmoid(z_t[0:H])               (write gate, one per head)
//   g_t   = -softplus(z_t[H:2H])            (log-decay, <= 0)
//   qhat  = q / ||q||  per (token, head)    (Algorithm 1's readout divides by ||q_t||; o is
//                                            linear in q, so the recurrence on qhat is that
//                                            readout; a zero query gives qhat = 0)
// x is read once for all heads, which is why this is its own kernel rather than part of the
// per-(chunk, head) preparation kernel (that would read each token's x once per head).
//
// bf16 with D % 64 == 0 and 2H in {16, 32, ..., 128}: one CTA per 128 tokens runs the
// projection on the tensor cores (tcgen05, M = 128 tokens, N = 2H, K = D in 64-wide steps
// through a 6-stage TMA ring) and the activations in the TMEM epilogue.  Other shapes and fp32:
// CUDA cores.  The query normalisation is a streaming kernel of its own (a group of Dk/8 lanes
// per row, 16-byte accesses), launched first on the same stream.
//
// Backward (CUDA cores): with dz = [deta * eta (1 - eta), dg * expm1(g)] (d(-softplus z)/dz =
// -sigmoid(z) = expm1(g)),  dx = dz W,  dW = dz^T x,  dbias = sum_t dz,
// dq = (dqhat - qhat (qhat . dqhat)) / ||q||.  dW and dbias are summed per 64-token tile into
// the workspace and then over tiles in a fixed order (deterministic).
#include <cuda.h>

#include <mutex>
#include <unordered_map>

#include "kla_device.cuh"
#include "kla_launch.h"
#include "kla_sm100.cuh"
#include "kla_tc_common.cuh"

namespace kla {

__device__ unsigned int g_gates_error = 0;

namespace {

using namespace sm100;

constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int GM = 128;    // tokens per CTA
constexpr int GKT = 64;    // K elements per stage (128 bytes of bf16)
constexpr int GST = 6;     // stages
constexpr int GTH = 192;   // threads: warps 0-3 epilogue, 4 loader, 5 MMA issuer

__device__ __forceinline__ float sigmoidf_(float z) { return 1.f / (1.f + __expf(-z)); }
__device__ __forceinline__ float softplusf_(float z) { return fmaxf(z, 0.f) + log1pf(__expf(-fabsf(z))); }

// Eight consecutive elements as fp32 and back (16 bytes of bf16, 32 of fp32).
__device__ __forceinline__ void ld8(const __nv_bfloat16* p, float* f) {
    unpack_bf16x8(*reinterpret_cast<const uint4*>(p), f);
}
__device__ __forceinline__ void ld8(const float* p, float* f) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void st8(__nv_bfloat16* p, const float* f) {
    uint4 w;
    w.x = pack_bf16x2(f[0], f[1]); w.y = pack_bf16x2(f[2], f[3]);
    w.z = pack_bf16x2(f[4], f[5]); w.w = pack_bf16x2(f[6], f[7]);
    *reinterpret_cast<uint4*>(p) = w;
}
__device__ __forceinline__ void st8(float* p, const float* f) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// qhat = q / ||q|| for every (token, head) row of Dk elements: a group of Dk / 8 lanes per row,
// eight elements per lane, the sum of squares reduced inside the group.  Streams q once.
template <typename Tin, int DK>
__global__ void __launch_bounds__(256) qnorm_kernel(const Tin* __restrict__ q, Tin* __restrict__ qhat, size_t rows) {
    constexpr int G = DK / 8;
    const size_t gid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t row = gid / G;
    const bool live = row < rows;
    const size_t off = (live ? row : 0) * DK + (gid % G) * 8;
    float x[8];
    ld8(q + off, x);
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) s = fmaf(x[e], x[e], s);
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float inv = s > 0.f ? rsqrtf(s) : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] *= inv;
    if (live) st8(qhat + off, x);
}

// dq = (dqhat - qhat (qhat . dqhat)) / ||q|| per row (zero where q is zero), same layout.
template <typename Tin, int DK>
__global__ void __launch_bounds__(256) qnorm_bwd_kernel(const Tin* __restrict__ q, const float* __restrict__ dqhat,
                                                        float* __restrict__ dq, size_t rows) {
    constexpr int G = DK / 8;
    const size_t gid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t row = gid / G;
    const bool live = row < rows;
    const size_t off = (live ? row : 0) * DK + (gid % G) * 8;
    float x[8], d[8];
    ld8(q + off, x);
    ld8(dqhat + off, d);
    float s = 0.f, p = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        s = fmaf(x[e], x[e], s);
        p = fmaf(x[e], d[e], p);
    }
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) {
        s += __shfl_xor_sync(0xffffffffu, s, o);
        p += __shfl_xor_sync(0xffffffffu, p, o);
    }
    const float inv = s > 0.f ? rsqrtf(s) : 0.f;  // 1 / ||q||;  qhat . dqhat = p / ||q||
    const float c = inv * inv * p;
#pragma unroll
    for (int e = 0; e < 8; ++e) d[e] = inv * (d[e] - x[e] * c);
    if (live) st8(dq + off, d);
}

template <typename Tin>
cudaError_t launch_qnorm(const Tin* q, Tin* qhat, size_t rows, int Dk, cudaStream_t st) {
    const size_t threads = rows * (size_t)(Dk / 8);
    const unsigned grid = (unsigned)((threads + 255) / 256);
    if (Dk == 128)
        qnorm_kernel<Tin, 128><<<grid, 256, 0, st>>>(q, qhat, rows);
    else
        qnorm_kernel<Tin, 64><<<grid, 256, 0, st>>>(q, qhat, rows);
    return cudaGetLastError();
}
template <typename Tin>
cudaError_t launch_qnorm_bwd(const Tin* q, const float* dqhat, float* dq, size_t rows, int Dk, cudaStream_t st) {
    const size_t threads = rows * (size_t)(Dk / 8);
    const unsigned grid = (unsigned)((threads + 255) / 256);
    if (Dk == 128)
        qnorm_bwd_kernel<Tin, 128><<<grid, 256, 0, st>>>(q, dqhat, dq, rows);
    else
        qnorm_bwd_kernel<Tin, 64><<<grid, 256, 0, st>>>(q, dqhat, dq, rows);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------
// Tensor-core projection (bf16).  Stage s: x tile [128 tokens x 64] (16 KB) then the W tile
// [NW rows x 64] (NW * 128 bytes, rounded up to 1 KB), both K-major with the 128-byte swizzle.
// ------------------------------------------------------------------------------------
struct GateBars {
    uint64_t full[GST], empty[GST], done;
    uint32_t tmem_base;
};

__global__ void __launch_bounds__(GTH, 1)
    gate_prologue_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                            const float* __restrict__ bias, float* __restrict__ eta, float* __restrict__ g, int N,
                            int D, int H, uint32_t w_bytes, uint32_t tmem_cols) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t stage_bytes = 16384 + w_bytes;
    GateBars* bars = reinterpret_cast<GateBars*>(sm + GST * stage_bytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NW = 2 * H, KT = D / GKT;
    const int tok0 = blockIdx.x * GM;
    const int ntok = min(GM, N - tok0);
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        for (int s = 0; s < GST; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->done), 1);
        fence_mbar_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_w);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&bars->tmem_base), tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    bool ok = true;

    if (warp == 4) {
        if (lane == 0) {  // loader
            for (int kt = 0; kt < KT && ok; ++kt) {
                const int s = kt % GST;
                if (kt >= GST) ok = mbar_wait_bounded(smem_u32(&bars->empty[s]), ((kt / GST) - 1) & 1, kWaitNs);
                if (!ok) break;
                const uint32_t full = smem_u32(&bars->full[s]);
                mbar_expect_tx(full, 16384 + (uint32_t)NW * 128);
                tma_load_2d(sbase + s * stage_bytes, &tm_x, full, kt * GKT, tok0);
                tma_load_2d(sbase + s * stage_bytes + 16384, &tm_w, full, kt * GKT, 0);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {  // MMA issuer: Z[token][j] = sum_k x[token][k] W[j][k]
            const uint32_t idesc = idesc_bf16(GM, NW, false, false);
            for (int kt = 0; kt < KT && ok; ++kt) {
                const int s = kt % GST;
                ok = mbar_wait_bounded(smem_u32(&bars->full[s]), (kt / GST) & 1, kWaitNs);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a = sbase + s * stage_bytes, bw = a + 16384;
#pragma unroll
                for (int k = 0; k < GKT / 16; ++k)
                    mma_bf16(tmem, smem_desc(a + 32 * k, 16, 1024), smem_desc(bw + 32 * k, 16, 1024), idesc,
                             (kt | k) > 0);
                mma_commit(smem_u32(&bars->empty[s]));
            }
            mma_commit(smem_u32(&bars->done));
        }
    }
    if (warp < 4) {  // epilogue: lane = token
        const bool got = mbar_wait_bounded(smem_u32(&bars->done), 0, kWaitNs);
        if (__any_sync(0xffffffffu, !got)) {
            ok = false;
        } else {
            tc_fence_after();
            const int t = 32 * warp + lane;
            const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
            for (int c0 = 0; c0 < NW; c0 += 16) {
                uint32_t z[16];
                tmem_ld16u(tmem + lane_base + c0, z);
                tmem_ld_wait();
                if (t < ntok) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int j = c0 + e;
                        const float zz = __uint_as_float(z[e]) + bias[j];
                        if (j < H)
                            eta[(size_t)(tok0 + t) * H + j] = sigmoidf_(zz);
                        else
                            g[(size_t)(tok0 + t) * H + (j - H)] = -softplusf_(zz);
                    }
                }
            }
        }
    }
    if (!ok) atomicOr(&g_gates_error, 1u);
    tc_fence_before();
    __syncthreads();
    // a stage that never completed leaves no copy in flight: the loader stops before issuing
    // past an expired wait, and every issued copy completes its own barrier
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols);
    }
}

// ------------------------------------------------------------------------------------
// CUDA-core projection: one warp per token, outputs in groups of 8.
// ------------------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(256) gate_prologue_simt_kernel(const Tin* __restrict__ x, const Tin* __restrict__ W,
                                                                 const float* __restrict__ bias, float* __restrict__ eta,
                                                                 float* __restrict__ g, int N, int D, int H) {
    const int lane = threadIdx.x & 31;
    const size_t t = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= (size_t)N) return;
    const int NW = 2 * H;
    const Tin* xr = x + t * D;
    for (int j0 = 0; j0 < NW; j0 += 8) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int d = lane; d < D; d += 32) {
            const float xv = to_f32(xr[d]);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (j0 + e < NW) acc[e] = fmaf(xv, to_f32(W[(size_t)(j0 + e) * D + d]), acc[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = warp_sum(acc[e]);
        if (lane < 8 && j0 + lane < NW) {
            float zz = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (e == lane) zz = acc[e];
            const int j = j0 + lane;
            zz += bias[j];
            if (j < H)
                eta[t * H + j] = sigmoidf_(zz);
            else
                g[t * H + (j - H)] = -softplusf_(zz);
        }
    }
}

// ------------------------------------------------------------------------------------
// Backward, per tile of 64 tokens: dz to shared memory; dx = dz W; partial dW, dbias of the
// tile to the workspace; dq from dqhat.
// ------------------------------------------------------------------------------------
constexpr int BT = 64;    // tokens per tile
constexpr int BD = 128;   // x / W columns per pass

template <typename Tin>
__global__ void __launch_bounds__(256) gate_bwd_tile_kernel(const Tin* __restrict__ x, const Tin* __restrict__ W,
                                                            const float* __restrict__ eta, const float* __restrict__ g,
                                                            const float* __restrict__ deta, const float* __restrict__ dg,
                                                            float* __restrict__ dx, float* __restrict__ part_w,
                                                            float* __restrict__ part_b, int N, int D, int H) {
    // one CTA per (64-token tile, 128-column block of D)
    extern __shared__ float smf[];
    const int NW = 2 * H;
    float* dz = smf;                   // [BT][NW]
    float* xs = dz + BT * NW;          // [BT][BD + 1]
    float* wsh = xs + BT * (BD + 1);   // [NW][BD + 1]
    const int tid = threadIdx.x;
    const int tile = blockIdx.x, d0 = blockIdx.y * BD;
    const int t0 = tile * BT;
    const int nt = min(BT, N - t0);
    const int nd = min(BD, D - d0);
    for (int i = tid; i < BT * NW; i += 256) {
        const int t = i / NW, j = i % NW;
        float v = 0.f;
        if (t < nt) {
            const size_t o = (size_t)(t0 + t) * H;
            if (j < H) {
                const float e = eta[o + j];
                v = deta[o + j] * e * (1.f - e);
            } else {
                v = dg[o + j - H] * expm1f(g[o + j - H]);
            }
        }
        dz[i] = v;
    }
    // eight elements per access (D % 8 == 0, so a group of eight is either in range or not)
    for (int i = tid; i < BT * (BD / 8); i += 256) {
        const int t = i / (BD / 8), c8 = 8 * (i % (BD / 8));
        float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (t < nt && c8 < nd) ld8(x + (size_t)(t0 + t) * D + d0 + c8, f);
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[t * (BD + 1) + c8 + e] = f[e];
    }
    for (int i = tid; i < NW * (BD / 8); i += 256) {
        const int j = i / (BD / 8), c8 = 8 * (i % (BD / 8));
        float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (c8 < nd) ld8(W + (size_t)j * D + d0 + c8, f);
#pragma unroll
        for (int e = 0; e < 8; ++e) wsh[j * (BD + 1) + c8 + e] = f[e];
    }
    __syncthreads();
    if (blockIdx.y == 0 && tid < NW) {  // dbias partial, fixed order over the tile's tokens
        float s = 0.f;
        for (int t = 0; t < BT; ++t) s += dz[t * NW + tid];
        part_b[(size_t)tile * NW + tid] = s;
    }
    // thread = column c (128) x half th; NW = 2H is even, so dz rows are read two gates at a time
    const int c = tid & (BD - 1), th = tid >> 7;
    // dx[t][c] = sum_j dz[t][j] W[j][c] for the thread's tokens t = th + 2 m: W's column held in
    // registers 16 gates at a time, dz rows broadcast
    {
        float acc[BT / 2];
#pragma unroll
        for (int m = 0; m < BT / 2; ++m) acc[m] = 0.f;
        for (int jb = 0; jb < NW; jb += 16) {
            float wr[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) wr[e] = (jb + e < NW) ? wsh[(jb + e) * (BD + 1) + c] : 0.f;
#pragma unroll
            for (int m = 0; m < BT / 2; ++m) {
                const float* zr = dz + (th + 2 * m) * NW + jb;
                float s = acc[m];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    if (jb + e < NW) {
                        const float2 z2 = *reinterpret_cast<const float2*>(zr + e);
                        s = fmaf(z2.x, wr[e], s);
                        s = fmaf(z2.y, wr[e + 1], s);
                    }
                }
                acc[m] = s;
            }
        }
        if (c < nd) {
#pragma unroll
            for (int m = 0; m < BT / 2; ++m) {
                const int t = th + 2 * m;
                if (t < nt) dx[(size_t)(t0 + t) * D + d0 + c] = acc[m];
            }
        }
    }
    // dW partial [j][c] = sum_t dz[t][j] x[t][c]: the thread's gates j = th (mod 2), eight at a time
    for (int jb = th * 8; jb < NW; jb += 16) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int t = 0; t < BT; ++t) {
            const float xv = xs[t * (BD + 1) + c];
            const float* zr = dz + t * NW + jb;
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                if (jb + e < NW) {
                    const float2 z2 = *reinterpret_cast<const float2*>(zr + e);
                    acc[e] = fmaf(z2.x, xv, acc[e]);
                    acc[e + 1] = fmaf(z2.y, xv, acc[e + 1]);
                }
            }
        }
        if (c < nd) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (jb + e < NW) part_w[((size_t)tile * NW + jb + e) * D + d0 + c] = acc[e];
        }
    }
}

// dW[j][d] = sum over tiles (fixed order), dbias[j] likewise.
// dW and dbias: the tiles' partial sums added in a fixed order.  A block takes 64 outputs; its
// four thread groups each sum a quarter of the tiles in order, then the quarters are added in
// order, so the result does not depend on scheduling.
constexpr int RED_OUT = 64, RED_PARTS = 4;
__global__ void __launch_bounds__(RED_OUT * RED_PARTS)
    gate_bwd_reduce_kernel(const float* __restrict__ part_w, const float* __restrict__ part_b, float* __restrict__ dW,
                           float* __restrict__ db, int ntile, int NW, int D) {
    __shared__ float sums[RED_PARTS][RED_OUT];
    const int p = threadIdx.x / RED_OUT, o = threadIdx.x % RED_OUT;
    const size_t i = (size_t)blockIdx.x * RED_OUT + o;
    const size_t total = (size_t)NW * D;
    const int per = (ntile + RED_PARTS - 1) / RED_PARTS, ta = p * per, tb = min(ntile, ta + per);
    float s = 0.f;
    if (i < total)
        for (int t = ta; t < tb; ++t) s += part_w[(size_t)t * total + i];
    sums[p][o] = s;
    __syncthreads();
    if (p == 0 && i < total) dW[i] = ((sums[0][o] + sums[1][o]) + sums[2][o]) + sums[3][o];
    if (blockIdx.x == 0 && p == 0) {
        for (int j = o; j < NW; j += RED_OUT) {
            float sb = 0.f;
            for (int t = 0; t < ntile; ++t) sb += part_b[(size_t)t * NW + j];
            db[j] = sb;
        }
    }
}

bool gate_tc_shape(const GateArgs& a) {
    return a.bf16 && a.D % GKT == 0 && a.H % 8 == 0 && 2 * a.H <= 256 && a.N >= 1;
}

}  // namespace

size_t gate_bwd_workspace(int N, int D, int H) {
    const size_t ntile = ((size_t)N + BT - 1) / BT;
    return ntile * 2 * H * ((size_t)D + 1) * sizeof(float);
}

namespace {
// The query normalisation shares no data with the gate projection (nor, in the backward, with
// the dx / dW kernels), so it runs on a second stream of the device beside them: the projection
// launches fewer CTAs than there are SMs.  The caller's stream waits for both before anything
// after the call.
cudaError_t side_stream(cudaStream_t* out) {
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

// Runs `side_work` on the side stream after everything already queued on st, and `main_work`
// on st; st then waits for the side stream.  Falls back to st alone if a side stream cannot be
// had.  The side work is always joined back, whatever either part returns.
template <typename FS, typename FM>
cudaError_t run_beside(cudaStream_t st, FS side_work, FM main_work) {
    cudaStream_t side = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    cudaError_t e = side_stream(&side);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_join, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(ev_fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side, ev_fork, 0);
    if (e != cudaSuccess) {
        if (ev_fork) cudaEventDestroy(ev_fork);
        if (ev_join) cudaEventDestroy(ev_join);
        e = side_work(st);
        return e == cudaSuccess ? main_work(st) : e;
    }
    e = side_work(side);
    const cudaError_t er = cudaEventRecord(ev_join, side);
    const cudaError_t em = e == cudaSuccess ? main_work(st) : e;
    const cudaError_t ej = er == cudaSuccess ? cudaStreamWaitEvent(st, ev_join, 0) : er;
    cudaEventDestroy(ev_fork);  // released once the work that uses them is done
    cudaEventDestroy(ev_join);
    return em != cudaSuccess ? em : ej;
}

cudaError_t launch_gates_only(const GateArgs& a, cudaStream_t st);
}  // namespace

cudaError_t launch_gate_prologue(const GateArgs& a, cudaStream_t st) {
    if (a.N == 0) return cudaSuccess;
    if (a.q == nullptr) return launch_gates_only(a, st);
    const size_t rows = (size_t)a.N * a.H;
    auto qn = [&](cudaStream_t s) {
        return a.bf16 ? launch_qnorm(static_cast<const __nv_bfloat16*>(a.q), static_cast<__nv_bfloat16*>(a.qhat), rows,
                                     a.Dk, s)
                      : launch_qnorm(static_cast<const float*>(a.q), static_cast<float*>(a.qhat), rows, a.Dk, s);
    };
    return run_beside(st, qn, [&](cudaStream_t s) { return launch_gates_only(a, s); });
}

namespace {
cudaError_t launch_gates_only(const GateArgs& a, cudaStream_t st) {
    if (gate_tc_shape(a)) {
        EncodeTiledFn enc = get_encode_fn();
        if (enc != nullptr) {
            const int NW = 2 * a.H;
            CUtensorMap mx, mw;
            const cuuint64_t dx[2] = {(cuuint64_t)a.D, (cuuint64_t)a.N};
            const cuuint64_t sx[1] = {(cuuint64_t)a.D * 2};
            const cuuint32_t bx[2] = {GKT, GM};
            const cuuint64_t dw[2] = {(cuuint64_t)a.D, (cuuint64_t)NW};
            const cuuint32_t bw[2] = {GKT, (cuuint32_t)NW};
            const cuuint32_t es[2] = {1, 1};
            if (enc(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.x), dx, sx, bx, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
                enc(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.W), dw, sx, bw, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
            const uint32_t w_bytes = ((uint32_t)NW * 128 + 1023) & ~1023u;
            uint32_t cols = 32;
            while (cols < (uint32_t)NW) cols <<= 1;
            const size_t smem = 1024 + GST * (16384 + (size_t)w_bytes) + sizeof(GateBars);
            cudaError_t e = cudaFuncSetAttribute(gate_prologue_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
            if (e != cudaSuccess) return e;
            gate_prologue_tc_kernel<<<(a.N + GM - 1) / GM, GTH, smem, st>>>(mx, mw, a.bias, a.eta, a.g, a.N, a.D,
                                                                            a.H, w_bytes, cols);
            return cudaGetLastError();
        }
    }
    const unsigned grid = (unsigned)(((size_t)a.N + 7) / 8);
    if (a.bf16)
        gate_prologue_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(a.x), static_cast<const __nv_bfloat16*>(a.W), a.bias, a.eta, a.g, a.N,
            a.D, a.H);
    else
        gate_prologue_simt_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(a.x),
                                                                static_cast<const float*>(a.W), a.bias, a.eta, a.g,
                                                                a.N, a.D, a.H);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_gate_prologue_bwd(const GateBwdArgs& a, void* ws, cudaStream_t st) {
    if (a.N == 0) {
        cudaError_t e = cudaMemsetAsync(a.dW, 0, (size_t)2 * a.H * a.D * sizeof(float), st);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.db, 0, (size_t)2 * a.H * sizeof(float), st);
        return e;
    }
    const int NW = 2 * a.H;
    const int ntile = (a.N + BT - 1) / BT;
    float* part_w = static_cast<float*>(ws);
    float* part_b = part_w + (size_t)ntile * NW * a.D;
    const size_t smem = sizeof(float) * ((size_t)BT * NW + (size_t)BT * (BD + 1) + (size_t)NW * (BD + 1));
    // dx and the dW / dbias partials, then their fixed-order reduction
    auto dxw = [&](cudaStream_t s) {
        cudaError_t e;
        if (a.bf16) {
            e = cudaFuncSetAttribute(gate_bwd_tile_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem);
            if (e != cudaSuccess) return e;
            gate_bwd_tile_kernel<__nv_bfloat16><<<dim3(ntile, (a.D + BD - 1) / BD), 256, smem, s>>>(
                static_cast<const __nv_bfloat16*>(a.x), static_cast<const __nv_bfloat16*>(a.W), a.eta, a.g, a.deta,
                a.dg, a.dx, part_w, part_b, a.N, a.D, a.H);
        } else {
            e = cudaFuncSetAttribute(gate_bwd_tile_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem);
            if (e != cudaSuccess) return e;
            gate_bwd_tile_kernel<float><<<dim3(ntile, (a.D + BD - 1) / BD), 256, smem, s>>>(
                static_cast<const float*>(a.x), static_cast<const float*>(a.W), a.eta, a.g, a.deta, a.dg, a.dx, part_w,
                part_b, a.N, a.D, a.H);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const size_t total = (size_t)NW * a.D;
        gate_bwd_reduce_kernel<<<(unsigned)((total + RED_OUT - 1) / RED_OUT), RED_OUT * RED_PARTS, 0, s>>>(
            part_w, part_b, a.dW, a.db, ntile, NW, a.D);
        return cudaGetLastError();
    };
    if (a.q == nullptr) return dxw(st);
    const size_t rows = (size_t)a.N * a.H;
    auto qn = [&](cudaStream_t s) {
        return a.bf16 ? launch_qnorm_bwd(static_cast<const __nv_bfloat16*>(a.q), a.dqhat, a.dq, rows, a.Dk, s)
                      : launch_qnorm_bwd(static_cast<const float*>(a.q), a.dqhat, a.dq, rows, a.Dk, s);
    };
    return run_beside(st, qn, dxw);
}

cudaError_t gates_take_error(cudaStream_t st, unsigned int* flag) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(flag, g_gates_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_gates_error, &zero, sizeof(unsigned int));
}

}  // namespace kla
