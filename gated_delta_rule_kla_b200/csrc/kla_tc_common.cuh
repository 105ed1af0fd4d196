// kla_tc_common.cuh -- pieces shared by the tensor-core chunk kernels: sizes, the blocked
// 64x64 unit-lower-triangular inverse, swizzled bf16 tile writers and the TMA map builder.
#pragma once

#include <cuda.h>

#include "kla_sm100.cuh"

namespace kla {

// cuTensorMapEncodeTiled, fetched from the driver at run time (null when there is no driver).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_fn();
// 4-D map over a [B, T, H, 128] bf16 tensor; box = 64 tokens x 64 features of one (b, h),
// 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H);

namespace tcc {

using namespace sm100;

constexpr int DK = 128, DV = 128, CH = 64;
constexpr int LDL = 68;  // row stride (floats) of the fp32 L/T buffer, 16-B rows

__device__ __forceinline__ size_t tok_index(int b, int t, int h, int T, int H) {
    return ((size_t)b * T + t) * H + h;
}

// Off-diagonal 16x16 block (I, J), I > J, of T in the Toff buffer: blocks ordered by
// distance d = I - J, then by J: (1,0) (2,1) (3,2) (2,0) (3,1) (3,0).
__device__ __forceinline__ int toff_block(int I, int J) {
    const int d = I - J;
    return (d == 1 ? 0 : (d == 2 ? 3 : 5)) + J;
}

// T = (I + L)^{-1} of the unit lower-triangular 64x64 matrix of Eq. (7), by blockwise
// forward substitution (Appendix B.2) on 16x16 blocks.  L: fp32, rows of LDL floats,
// strictly lower (upper part zero).
//   diagonal blocks  D_I = (I + L_II)^{-1}: column by column (64 threads), written over L_II
//   off-diagonal     T_IJ = -D_I sum_{K=J}^{I-1} L_IK T_KJ (T_JJ = D_J), by distance
//                    d = I - J = 1, 2, 3, into Toff (6 blocks of 16x16); L stays intact.
// X is scratch for 3 x 256 floats.  All NT threads of the CTA must call it.
template <int NT>
__device__ __forceinline__ void invert_unit_lower64(float* Lf, float* Toff, float* X, int tid) {
    if (tid < 64) {
        const int base = 16 * (tid >> 4), l = tid & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int j = 0; j + 1 < i; j += 2) {
                a0 = fmaf(Lf[(base + i) * LDL + base + j], x[j], a0);
                a1 = fmaf(Lf[(base + i) * LDL + base + j + 1], x[j + 1], a1);
            }
            if (i & 1) a0 = fmaf(Lf[(base + i) * LDL + base + i - 1], x[i - 1], a0);
            x[i] = (i < l) ? 0.f : ((i == l) ? 1.f : -(a0 + a1));
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 16; ++i) Lf[(base + i) * LDL + base + l] = x[i];
    }
    __syncthreads();
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
        const int njobs = 64 * (4 - d);  // (block, row, column quad)
        for (int job = tid; job < njobs; job += NT) {
            const int J = job >> 6, I = J + d, r = (job >> 2) & 15, cq = job & 3;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int K = J; K < I; ++K) {
                const float* tk = (K == J) ? (Lf + 16 * J * LDL + 16 * J) : (Toff + toff_block(K, J) * 256);
                const int ldt = (K == J) ? LDL : 16;
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float l = Lf[(16 * I + r) * LDL + 16 * K + m];
                    const float4 t = *reinterpret_cast<const float4*>(tk + m * ldt + 4 * cq);
                    acc.x = fmaf(l, t.x, acc.x);
                    acc.y = fmaf(l, t.y, acc.y);
                    acc.z = fmaf(l, t.z, acc.z);
                    acc.w = fmaf(l, t.w, acc.w);
                }
            }
            *reinterpret_cast<float4*>(X + job * 4) = acc;
        }
        __syncthreads();
        for (int job = tid; job < njobs; job += NT) {
            const int J = job >> 6, I = J + d, r = (job >> 2) & 15, cq = job & 3;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float l = Lf[(16 * I + r) * LDL + 16 * I + m];  // D_I
                const float4 x = *reinterpret_cast<const float4*>(X + ((J << 6) + (m << 2) + cq) * 4);
                acc.x = fmaf(l, x.x, acc.x);
                acc.y = fmaf(l, x.y, acc.y);
                acc.z = fmaf(l, x.z, acc.z);
                acc.w = fmaf(l, x.w, acc.w);
            }
            *reinterpret_cast<float4*>(Toff + toff_block(I, J) * 256 + r * 16 + 4 * cq) =
                make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
        }
        __syncthreads();
    }
}

// T = (I + L)^{-1} of the unit lower-triangular 64x64 matrix of Eq. (7), in place, by
// recursive doubling on the block form of the inverse (a rearrangement of the forward
// substitution of Appendix B.2):
//   [A 0; C B]^{-1} = [A^{-1} 0; -B^{-1} C A^{-1}  B^{-1}].
// Level 0 inverts the eight 8x8 diagonal blocks by substitution (64 threads); levels 8, 16, 32
// then join pairs of inverted s x s blocks, writing -T_B (L_BA T_A) over L_BA, with every thread
// computing PER = 32 s / NT adjacent outputs of each product.  On entry Lf holds L (rows of
// LDL floats, zero on and above the diagonal); on exit it holds T, ones on the diagonal.
// X is scratch for 1024 floats.  All NT (= 256) threads of the CTA must call it.
template <int S, int NT>
__device__ __forceinline__ void inverse_join_level(float* Lf, float* X, int tid) {
    constexpr int PER = 32 * S / NT;  // outputs per thread: 1, 2, 4 for S = 8, 16, 32
    static_assert(PER >= 1 && PER <= 4 && S % PER == 0, "join level shape");
    const int idx = tid * PER;
    const int p = idx / (S * S), rem = idx % (S * S), i = rem / S, j0 = rem % S;
    const int A0 = 2 * S * p, B0 = A0 + S;
    // PER adjacent floats at a 4*PER-byte aligned address (rows of LDL = 68 floats, j0 a
    // multiple of PER, block offsets multiples of 8): one vector load.
    auto ld = [](const float* p, float (&v)[PER]) {
        if constexpr (PER == 4) {
            const float4 t = *reinterpret_cast<const float4*>(p);
            v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
        } else if constexpr (PER == 2) {
            const float2 t = *reinterpret_cast<const float2*>(p);
            v[0] = t.x; v[1] = t.y;
        } else {
            v[0] = *p;
        }
    };
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    // X_p = L_BA T_A   (T_A lower triangular: zero above its diagonal)
    const float* lrow = Lf + (B0 + i) * LDL;
#pragma unroll 8
    for (int k = 0; k < S; ++k) {
        const float l = lrow[A0 + k];
        float t[PER];
        ld(Lf + (A0 + k) * LDL + A0 + j0, t);
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = fmaf(l, t[e], acc[e]);
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) X[idx + e] = acc[e];
    __syncthreads();
    // T_BA = -T_B X_p, over L_BA (whose reads are all done)
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
#pragma unroll 8
    for (int k = 0; k < S; ++k) {
        const float l = lrow[B0 + k];
        float x[PER];
        ld(X + p * S * S + k * S + j0, x);
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = fmaf(l, x[e], acc[e]);
    }
    float* dst = Lf + (B0 + i) * LDL + A0 + j0;
    if constexpr (PER == 4) {
        *reinterpret_cast<float4*>(dst) = make_float4(-acc[0], -acc[1], -acc[2], -acc[3]);
    } else if constexpr (PER == 2) {
        *reinterpret_cast<float2*>(dst) = make_float2(-acc[0], -acc[1]);
    } else {
        dst[0] = -acc[0];
    }
    __syncthreads();
}

// Join levels 16 and 32 with the triangles' zeros skipped.  The same sums as
// inverse_join_level, term for term and in the same order (only products with a structural
// zero factor are left out, so the results are bit-identical), with warp-uniform trip counts:
// phase 1 (X = L_BA T_A, T_A[k][j] = 0 for k < j) gives each warp a group of columns j0.. and
// runs k from j0; phase 2 (T_BA = -T_B X, T_B[i][k] = 0 for k > i) gives each warp a group of
// rows and stops after the group's last row.  Operand rows are read as float4 (k four at a
// time; every bound is a multiple of 4).  256 threads.
__device__ __forceinline__ void inverse_join32_tri(float* Lf, float* X, int tid) {
    const int w = tid >> 5, lane = tid & 31;
    {  // warp w: columns 4w .. 4w + 3 of X, lane: row i
        const int i = lane, j0 = 4 * w;
        const float* lrow = Lf + (32 + i) * LDL;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        for (int k = j0; k < 32; k += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lrow + k);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float4 t = *reinterpret_cast<const float4*>(Lf + (k + u) * LDL + j0);
                a0 = fmaf(lv[u], t.x, a0);
                a1 = fmaf(lv[u], t.y, a1);
                a2 = fmaf(lv[u], t.z, a2);
                a3 = fmaf(lv[u], t.w, a3);
            }
        }
        *reinterpret_cast<float4*>(X + i * 32 + j0) = make_float4(a0, a1, a2, a3);
    }
    __syncthreads();
    {  // warp w: rows 4w .. 4w + 3 of T_BA, lane: column j
        const int j = lane, i0 = 4 * w;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < i0 + 4; k += 4) {
            float tb[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float4 t = *reinterpret_cast<const float4*>(Lf + (32 + i0 + r) * LDL + 32 + k);
                tb[r][0] = t.x; tb[r][1] = t.y; tb[r][2] = t.z; tb[r][3] = t.w;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float x = X[(k + u) * 32 + j];
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[r] = fmaf(tb[r][u], x, acc[r]);
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) Lf[(32 + i0 + r) * LDL + j] = -acc[r];
    }
    __syncthreads();
}

__device__ __forceinline__ void inverse_join16_tri(float* Lf, float* X, int tid) {
    const int w = tid >> 5, lane = tid & 31;
    const int p = w >> 2, A0 = 32 * p, B0 = A0 + 16;
    {  // warp: join p, columns 4 (w & 3) .. + 3; lane: row lane & 15, column pair lane >> 4
        const int i = lane & 15, j0 = 4 * (w & 3), jc = j0 + 2 * (lane >> 4);
        const float* lrow = Lf + (B0 + i) * LDL + A0;
        float a0 = 0.f, a1 = 0.f;
        for (int k = j0; k < 16; k += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lrow + k);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 t = *reinterpret_cast<const float2*>(Lf + (A0 + k + u) * LDL + A0 + jc);
                a0 = fmaf(lv[u], t.x, a0);
                a1 = fmaf(lv[u], t.y, a1);
            }
        }
        *reinterpret_cast<float2*>(X + p * 256 + i * 16 + jc) = make_float2(a0, a1);
    }
    __syncthreads();
    {  // warp: join p, rows 4 (w & 3) .. + 3; lane: column lane & 15, row pair lane >> 4
        const int j = lane & 15, i0 = 4 * (w & 3), ir = i0 + 2 * (lane >> 4);
        float c0 = 0.f, c1 = 0.f;
        for (int k = 0; k < i0 + 4; k += 4) {
            const float4 t0 = *reinterpret_cast<const float4*>(Lf + (B0 + ir) * LDL + B0 + k);
            const float4 t1 = *reinterpret_cast<const float4*>(Lf + (B0 + ir + 1) * LDL + B0 + k);
            const float r0[4] = {t0.x, t0.y, t0.z, t0.w}, r1[4] = {t1.x, t1.y, t1.z, t1.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float x = X[p * 256 + (k + u) * 16 + j];
                c0 = fmaf(r0[u], x, c0);
                c1 = fmaf(r1[u], x, c1);
            }
        }
        Lf[(B0 + ir) * LDL + A0 + j] = -c0;
        Lf[(B0 + ir + 1) * LDL + A0 + j] = -c1;
    }
    __syncthreads();
}

template <int NT>
__device__ __forceinline__ void invert_unit_lower64_doubling(float* Lf, float* X, int tid) {
    static_assert(NT == 256, "the join levels assume 256 threads");
    if (tid < 64) {  // 8x8 diagonal block tid / 8, column tid % 8
        const int base = 8 * (tid >> 3), c = tid & 7;
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) s = fmaf(Lf[(base + i) * LDL + base + j], x[j], s);
            x[i] = (i < c) ? 0.f : ((i == c) ? 1.f : -s);
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) Lf[(base + i) * LDL + base + c] = x[i];
    }
    __syncthreads();
    inverse_join_level<8, NT>(Lf, X, tid);
    inverse_join16_tri(Lf, X, tid);
    inverse_join32_tri(Lf, X, tid);
}

// Store the 16-byte chunks c and c + 1 (c even) of row r of a 128B-swizzled [rows x 64] bf16
// block in global memory with one 32-byte store: under the swizzle they are the two halves of
// one aligned 32-byte sector (physical chunks c ^ (r & 7) and that ^ 1), in either order.
// `block` must be 32-byte aligned.
__device__ __forceinline__ void st_pair_sw128_global(uint8_t* block, int r, int c, uint4 a, uint4 b) {
    const int p = c ^ (r & 7);
    uint8_t* dst = block + r * 128 + ((p & ~1) << 4);
    const uint4 f = (p & 1) ? b : a, g = (p & 1) ? a : b;
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(f.x), "r"(f.y),
                 "r"(f.z), "r"(f.w), "r"(g.x), "r"(g.y), "r"(g.z), "r"(g.w)
                 : "memory");
}

// bf16 hi/lo words of 8 fp32 values (one 16-byte chunk of each of the two blocks): per pair,
// the hi word is one paired rounding, the hi values are read back from its halves, and the
// remainders are rounded as a pair (hi = rn(x), lo = rn(x - hi), as split_bf16).
__device__ __forceinline__ uint32_t split_word2(float a, float b, uint32_t& lo) {
    const uint32_t hw = pack_bf16x2(a, b);
    lo = pack_bf16x2(a - __uint_as_float(hw << 16), b - __uint_as_float(hw & 0xffff0000u));
    return hw;
}
__device__ __forceinline__ void split_chunk8(const float* v, uint4& uh, uint4& ul) {
    uh.x = split_word2(v[0], v[1], ul.x);
    uh.y = split_word2(v[2], v[3], ul.y);
    uh.z = split_word2(v[4], v[5], ul.z);
    uh.w = split_word2(v[6], v[7], ul.w);
}

// Global versions of st_chunks_split / st_chunks_bf16 for an even count of chunks starting
// at an even chunk: 32-byte stores, whole sectors.
__device__ __forceinline__ void st_chunks_split_global(uint8_t* hi_block, uint8_t* lo_block, int r, int c0, int n,
                                                       const float* v) {
#pragma unroll
    for (int c = 0; c < n; c += 2) {
        uint4 h0, l0, h1, l1;
        split_chunk8(v + 8 * c, h0, l0);
        split_chunk8(v + 8 * c + 8, h1, l1);
        st_pair_sw128_global(hi_block, r, c0 + c, h0, h1);
        st_pair_sw128_global(lo_block, r, c0 + c, l0, l1);
    }
}
// Packed bf16 words (two features per word, lower feature in the low half) as pieces
// c0 .. c0 + n - 1 of row r of a 128-byte-swizzled global tile (c0 and n even).
__device__ __forceinline__ void st_words_sw128_global(uint8_t* block, int r, int c0, int n, const uint32_t* w) {
#pragma unroll
    for (int c = 0; c < n; c += 2)
        st_pair_sw128_global(block, r, c0 + c, make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]),
                             make_uint4(w[4 * c + 4], w[4 * c + 5], w[4 * c + 6], w[4 * c + 7]));
}
// A thread's 32 TMEM columns of packed bf16 hi and lo words (64 features of its lane) as one
// row of a global hi tile and the same row of the lo tile 'lo_off' bytes after it.
__device__ __forceinline__ void st_tmem_row_global(uint32_t t_hi, uint32_t t_lo, uint8_t* block, uint32_t lo_off,
                                                   int r) {
    float h[32], l[32];
    tmem_ld32(t_hi, h);
    tmem_ld32(t_lo, l);
    tmem_ld_wait();
    uint32_t wh[32], wl[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        wh[e] = __float_as_uint(h[e]);
        wl[e] = __float_as_uint(l[e]);
    }
    st_words_sw128_global(block, r, 0, 8, wh);
    st_words_sw128_global(block + lo_off, r, 0, 8, wl);
}
__device__ __forceinline__ void st_chunks_bf16_global(uint8_t* block, int r, int c0, int n, const float* v) {
#pragma unroll
    for (int c = 0; c < n; c += 2) {
        uint4 a, b;
        a.x = pack_bf16x2(v[8 * c + 0], v[8 * c + 1]); a.y = pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
        a.z = pack_bf16x2(v[8 * c + 4], v[8 * c + 5]); a.w = pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
        b.x = pack_bf16x2(v[8 * c + 8], v[8 * c + 9]); b.y = pack_bf16x2(v[8 * c + 10], v[8 * c + 11]);
        b.z = pack_bf16x2(v[8 * c + 12], v[8 * c + 13]); b.w = pack_bf16x2(v[8 * c + 14], v[8 * c + 15]);
        st_pair_sw128_global(block, r, c0 + c, a, b);
    }
}

// Write 32 tokens of one dk column, v[e] at token t0 + e, into a [64 tokens x 64 dk] x 2
// swizzled bf16 tile pair in shared memory (block dk / 64), from a warp whose consecutive
// lanes hold consecutive dk.  Lane pairs (dk even, dk + 1) trade values so that each lane
// writes whole 32-bit words (two dk of one token): of each token pair (t, t + 4) the even
// lane writes t and the odd lane t + 4, whose swizzled 64-byte runs use the other 16 banks.
__device__ __forceinline__ void st_w_tokens_smem(uint8_t* base, int dk, int t0, const float* v, int lane) {
    const int odd = lane & 1, dk0 = dk & ~1;
    uint8_t* blk = base + (dk0 >> 6) * 8192;
    const int col = dk0 & 63;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int e0 = (i & 3) + 8 * (i >> 2);  // 0..3, 8..11, 16..19, 24..27
        const float other = __shfl_xor_sync(0xffffffffu, odd ? v[e0] : v[e0 + 4], 1);
        const uint32_t w = odd ? pack_bf16x2(other, v[e0 + 4]) : pack_bf16x2(v[e0], other);
        const int t = t0 + e0 + 4 * odd;
        *reinterpret_cast<uint32_t*>(blk + t * 128 + (((col >> 3) ^ (t & 7)) << 4) + (col & 7) * 2) = w;
    }
}

// Write chunks [c0, c0 + n) of row r of a swizzled bf16 block from 8*n fp32 values.
__device__ __forceinline__ void st_chunks_bf16(uint8_t* block, int r, int c0, int n, const float* v) {
#pragma unroll
    for (int c = 0; c < n; ++c) {
        uint4 u;
        u.x = pack_bf16x2(v[8 * c + 0], v[8 * c + 1]);
        u.y = pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
        u.z = pack_bf16x2(v[8 * c + 4], v[8 * c + 5]);
        u.w = pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
        *reinterpret_cast<uint4*>(block + sw128_off(r, c0 + c)) = u;
    }
}

// Split 8*n fp32 values into hi/lo bf16 and write chunks [c0, c0 + n) of row r of two blocks.
__device__ __forceinline__ void st_chunks_split(uint8_t* hi_block, uint8_t* lo_block, int r, int c0, int n,
                                                const float* v) {
#pragma unroll
    for (int c = 0; c < n; ++c) {
        uint4 uh, ul;
        split_chunk8(v + 8 * c, uh, ul);
        *reinterpret_cast<uint4*>(hi_block + sw128_off(r, c0 + c)) = uh;
        *reinterpret_cast<uint4*>(lo_block + sw128_off(r, c0 + c)) = ul;
    }
}


// ---- per-chunk record of the split forward's preparation kernel (byte offsets in the
//      workspace); tiles use the 128-byte swizzle
constexpr uint32_t REC_W = 0;        // -W bf16: [64 tokens x 64 dk] x 2 blocks         16 KB
constexpr uint32_t REC_KT = 16384;   // Ktil hi: [64 tokens x 64 dk] x 2 blocks        16 KB
constexpr uint32_t REC_KTLO = 32768; // Ktil lo                                        16 KB
constexpr uint32_t REC_P = 49152;    // P hi [64 x 64], then P lo                       16 KB
constexpr uint32_t REC_TPP = 65536;  // T'' = T Diag(c) hi [64 x 64], then lo              16 KB
                                     // (the state pass forms U' = T'' V itself)
constexpr uint32_t REC_TILES = 81920;
constexpr uint32_t REC_SC = REC_TILES;  // gamma[64], gamma_last of the next chunk, of the previous chunk  512 B
constexpr uint32_t REC_SCB = 512;
constexpr size_t REC_BYTES = REC_TILES + REC_SCB;
// Diagonal gating: the scalars are the next chunk's per-channel decay Gam_last[128]; Q o Gam
// (one bf16 rounding, [64 tokens x 64 dk] x 2 blocks, swizzled) and the chunk's own
// Gam_last[128] follow.
constexpr uint32_t REC_QG = (uint32_t)REC_BYTES;                                //  16 KB
constexpr uint32_t REC_GL = REC_QG + 16384;                                     //  512 B
constexpr size_t REC_BYTES_D = REC_GL + 512;

// Split fp32 values into bf16 hi + lo words, two consecutive K indices per 32-bit word (the
// lower index in the low half): hi = rn(x), lo = rn(x - hi).
template <int N>
__device__ __forceinline__ void split_pack(const float* x, uint32_t* hp, uint32_t* lp) {
#pragma unroll
    for (int e = 0; e < N / 2; ++e) {
        const uint32_t hw = pack_bf16x2(x[2 * e], x[2 * e + 1]);
        hp[e] = hw;
        lp[e] = pack_bf16x2(x[2 * e] - __uint_as_float(hw << 16), x[2 * e + 1] - __uint_as_float(hw & 0xffff0000u));
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Raise the expected transaction bytes of the current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx_only(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Pack fp32 pairs into bf16 words (hi part only), the lower K index in the low half.
template <int N>
__device__ __forceinline__ void pack_hi(const float* x, uint32_t* hp) {
#pragma unroll
    for (int e = 0; e < N / 2; ++e) hp[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
}

// Epilogue warp: make this warp's TMEM stores visible to the MMA issuer, then arrive once.
__device__ __forceinline__ void epi_signal(uint32_t bar, int tid) {
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(bar);
}

}  // namespace tcc
}  // namespace kla
