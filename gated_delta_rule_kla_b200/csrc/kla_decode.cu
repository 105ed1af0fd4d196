// kla_decode.cu -- single-token KLA decode step ("Kaczmarz Linear Attention", Algorithm 1,
// left panel, lines 2-6), fp32 state updated in place.
//
// Each column j of S evolves on its own given (k, q, alpha, beta):
//   e_j  = v_j - alpha (S^T k)_j
//   S'_ij = alpha S_ij + beta k_i e_j
//   o_j  = (S'^T q)_j = alpha (S^T q)_j + beta (k.q) e_j
// so one pass that reads S once yields both reductions; the update is then applied to
// the registers already holding S and written back once.  The kernel is HBM bound:
// 2 * Dk * Dv * 4 bytes of state traffic per head against ~7 Dk Dv FLOPs.
//
// Mapping: one CTA per (b, h), 256 threads.  A thread owns 4 adjacent columns (one
// 16-byte vector) of DK/ROWG rows; a warp reads 32 consecutive float4 = one 512-byte
// contiguous row segment, so every load and store is fully coalesced.
#include "kla_device.cuh"
#include "kla_launch.h"

namespace kla {

template <int DK, int DV, typename Tin, typename TOut>
__global__ void __launch_bounds__(256) decode_step_kernel(const Tin* __restrict__ q,
                                                          const Tin* __restrict__ k,
                                                          const Tin* __restrict__ v,
                                                          const float* __restrict__ eta,
                                                          const float* __restrict__ g, float eps,
                                                          float* __restrict__ S,
                                                          TOut* __restrict__ o) {
    constexpr int NT = 256;
    constexpr int COLG = DV / 4;       // float4 column groups
    constexpr int ROWG = NT / COLG;    // row groups
    constexpr int RPT = DK / ROWG;     // rows per thread
    static_assert(NT % COLG == 0 && DK % ROWG == 0, "tile mapping");

    __shared__ float ks[DK], qs[DK];
    __shared__ float4 red_k[ROWG][COLG], red_q[ROWG][COLG];
    __shared__ float scal[2][8];

    const int head = blockIdx.x;  // b * H + h
    const int tid = threadIdx.x;
    const int cg = tid % COLG;
    const int rg = tid / COLG;

    // Issue the state loads first: they are the only large traffic.
    float4* Sh = reinterpret_cast<float4*>(S + (size_t)head * DK * DV);
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) s[r] = Sh[(size_t)(rg + r * ROWG) * COLG + cg];

    // k, q into shared memory; ||k||^2 and k.q reduced over the block.
    float kk = 0.f, kq = 0.f;
    for (int i = tid; i < DK; i += NT) {
        float kv = to_f32(k[(size_t)head * DK + i]);
        float qv = to_f32(q[(size_t)head * DK + i]);
        ks[i] = kv;
        qs[i] = qv;
        kk += kv * kv;
        kq += kv * qv;
    }
    kk = warp_sum(kk);
    kq = warp_sum(kq);
    if ((tid & 31) == 0) {
        scal[0][tid >> 5] = kk;
        scal[1][tid >> 5] = kq;
    }
    __syncthreads();
    float n2 = 0.f, kdq = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        n2 += scal[0][w];
        kdq += scal[1][w];
    }
    const float alpha = expf(g[head]);
    const float den = n2 + eps;
    const float beta = den > 0.f ? eta[head] / den : 0.f;

    // Partial S^T k and S^T q over this thread's rows.
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const float ki = ks[rg + r * ROWG];
        const float qi = qs[rg + r * ROWG];
        pk.x = fmaf(s[r].x, ki, pk.x); pk.y = fmaf(s[r].y, ki, pk.y);
        pk.z = fmaf(s[r].z, ki, pk.z); pk.w = fmaf(s[r].w, ki, pk.w);
        pq.x = fmaf(s[r].x, qi, pq.x); pq.y = fmaf(s[r].y, qi, pq.y);
        pq.z = fmaf(s[r].z, qi, pq.z); pq.w = fmaf(s[r].w, qi, pq.w);
    }
    red_k[rg][cg] = pk;
    red_q[rg][cg] = pq;
    __syncthreads();
    float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sq = sk;
#pragma unroll
    for (int w = 0; w < ROWG; ++w) {
        float4 a = red_k[w][cg], b = red_q[w][cg];
        sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
        sq.x += b.x; sq.y += b.y; sq.z += b.z; sq.w += b.w;
    }
    // e = v - alpha S^T k  (four columns of this thread)
    const Tin* vh = v + (size_t)head * DV + cg * 4;
    float4 e;
    e.x = to_f32(vh[0]) - alpha * sk.x;
    e.y = to_f32(vh[1]) - alpha * sk.y;
    e.z = to_f32(vh[2]) - alpha * sk.z;
    e.w = to_f32(vh[3]) - alpha * sk.w;
    float4 be = make_float4(beta * e.x, beta * e.y, beta * e.z, beta * e.w);

    // S <- alpha S + beta k e^T, written back in place.
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const float ki = ks[rg + r * ROWG];
        float4 x = s[r];
        x.x = fmaf(alpha, x.x, ki * be.x);
        x.y = fmaf(alpha, x.y, ki * be.y);
        x.z = fmaf(alpha, x.z, ki * be.z);
        x.w = fmaf(alpha, x.w, ki * be.w);
        Sh[(size_t)(rg + r * ROWG) * COLG + cg] = x;
    }
    // o = alpha S^T q + (k.q) beta e
    if (o != nullptr && rg == 0) {
        TOut* oh = o + (size_t)head * DV + cg * 4;
        oh[0] = from_f32<TOut>(fmaf(alpha, sq.x, kdq * be.x));
        oh[1] = from_f32<TOut>(fmaf(alpha, sq.y, kdq * be.y));
        oh[2] = from_f32<TOut>(fmaf(alpha, sq.z, kdq * be.z));
        oh[3] = from_f32<TOut>(fmaf(alpha, sq.w, kdq * be.w));
    }
}

template <int DK, int DV, typename Tin, typename TOut>
static cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t st) {
    decode_step_kernel<DK, DV, Tin, TOut><<<a.B * a.H, 256, 0, st>>>(
        static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
        a.eta, a.g, a.eps, a.S, static_cast<TOut*>(a.o));
    return cudaGetLastError();
}

template <int DK, int DV, typename Tin>
static cudaError_t launch_decode_o(const DecodeArgs& a, cudaStream_t st) {
    return a.out_bf16 ? launch_decode_t<DK, DV, Tin, __nv_bfloat16>(a, st)
                      : launch_decode_t<DK, DV, Tin, float>(a, st);
}

template <typename Tin>
static cudaError_t launch_decode_d(const DecodeArgs& a, cudaStream_t st) {
    if (a.Dk == 128 && a.Dv == 128) return launch_decode_o<128, 128, Tin>(a, st);
    if (a.Dk == 128 && a.Dv == 64) return launch_decode_o<128, 64, Tin>(a, st);
    if (a.Dk == 64 && a.Dv == 128) return launch_decode_o<64, 128, Tin>(a, st);
    return launch_decode_o<64, 64, Tin>(a, st);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
    if (a.bf16) return launch_decode_d<__nv_bfloat16>(a, st);
    return launch_decode_d<float>(a, st);
}

}  // namespace kla
