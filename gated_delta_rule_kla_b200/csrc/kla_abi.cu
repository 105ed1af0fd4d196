// kla_abi.cu -- the extern "C" boundary of libkla.so (declared in include/kla.h).
// Host-side validation, workspace layout and kernel dispatch; no device arithmetic here.
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <atomic>
#include <string>

#include "kla.h"
#include "kla_device.cuh"
#include "kla_launch.h"
#include "kla_tc_common.cuh"

namespace {

// Set by kla_debug_inject_wait_timeout, taken (and cleared) by the next kla_decode_step.
std::atomic<int> g_inject_timeout{0};

thread_local std::string g_last_error;

kla_status fail(kla_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
kla_status fail(kla_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

kla_status cuda_fail(cudaError_t e, const char* where) {
    return fail(KLA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// Workspaces take 32-byte stores (whole sectors of the swizzled tile images).
bool aligned32(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// KLA_BETA_DIRECT rides in a dtype argument: take it off (leaving the element type) and say
// whether it was set.  The kernels learn it as eps = kla::kBetaDirect, a value the checks
// below never let through otherwise.
bool take_beta_flag(int& dtype) {
    const bool direct = (dtype & KLA_BETA_DIRECT) != 0;
    dtype &= ~KLA_BETA_DIRECT;
    return direct;
}
float kernel_eps(float eps, bool direct) { return direct ? kla::kBetaDirect : eps; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

kla_status check_common(int B, int T, int H, int Dk, int Dv, int chunk, int dtype, int out_dtype,
                        float eps) {
    if (B < 1 || H < 1 || T < 0)
        return fail(KLA_ERR_INVALID_ARG, "sizes must satisfy B>=1, H>=1, T>=0 (got B=%d T=%d H=%d)",
                    B, T, H);
    if (!(eps >= 0.f)) return fail(KLA_ERR_INVALID_ARG, "eps must be >= 0 (got %g)", (double)eps);
    if ((Dk != 64 && Dk != 128) || (Dv != 64 && Dv != 128))
        return fail(KLA_ERR_UNSUPPORTED, "Dk, Dv must be 64 or 128 (got Dk=%d Dv=%d)", Dk, Dv);
    if (chunk != kla::kChunkLen)
        return fail(KLA_ERR_UNSUPPORTED, "chunk must be %d (got %d)", kla::kChunkLen, chunk);
    if (dtype != KLA_F32 && dtype != KLA_BF16)
        return fail(KLA_ERR_UNSUPPORTED, "dtype must be KLA_F32 or KLA_BF16 (got %d)", dtype);
    if (out_dtype != KLA_F32 && out_dtype != KLA_BF16)
        return fail(KLA_ERR_UNSUPPORTED, "out_dtype must be KLA_F32 or KLA_BF16 (got %d)", out_dtype);
    // 32-bit index headroom for per-token offsets inside kernels is not assumed: kernels
    // index with size_t; but B*H and grid sizes must fit the launch limits.
    if ((long long)B * H > (1LL << 30)) return fail(KLA_ERR_UNSUPPORTED, "B*H too large");
    return KLA_OK;
}

#define REQUIRE_PTR(p)                                                                    \
    do {                                                                                  \
        if ((p) == nullptr) return fail(KLA_ERR_INVALID_ARG, "%s must not be NULL", #p); \
        if (!aligned16(p)) return fail(KLA_ERR_INVALID_ARG, "%s must be 16-byte aligned", #p); \
    } while (0)
#define OPTIONAL_PTR(p)                                                                        \
    do {                                                                                       \
        if (!aligned16(p)) return fail(KLA_ERR_INVALID_ARG, "%s must be 16-byte aligned", #p); \
    } while (0)

// Shapes the tensor-core backward serves (bf16, Dk == Dv == 128).
bool tc_bwd_shape(int T, int Dk, int Dv, int dtype) {
    return dtype == KLA_BF16 && Dk == 128 && Dv == 128 && T >= 1;
}

// The backward (and the training forward) run on the tensor cores for their shapes when the
// workspace holds the tensor-core layout; the decision depends only on the arguments.
bool tc_bwd_path(int B, int T, int H, int Dk, int Dv, int dtype, size_t ws_bytes) {
    return tc_bwd_shape(T, Dk, Dv, dtype) && kla::get_encode_fn() != nullptr &&
           ws_bytes >= kla::chunk_bwd_tc_workspace(B, T, H, false);
}

// Diagonal-gated backward: [S at every internal chunk start | acc_dq | acc_dkh | acc_dG (per
// channel) | acc_db, acc_dc | the split forward's records]; the accumulators are zeroed on
// every call.
size_t diag_bwd_ws_layout(int B, int T, int H, int Dk, int Dv, size_t* off) {
    const size_t CDl = (size_t)kla::diag_chunk_len();
    const size_t NC = ((size_t)T + CDl - 1) / CDl;
    const size_t ntok = (size_t)B * T * H;
    size_t o = 0;
    off[0] = o;
    o += align256((size_t)B * H * NC * Dk * Dv * sizeof(float));
    off[1] = o;
    o += align256(ntok * Dk * sizeof(float));
    off[2] = o;
    o += align256(ntok * Dk * sizeof(float));
    off[3] = o;
    o += align256(ntok * Dk * sizeof(float));
    off[4] = o;
    o += align256(2 * ntok * sizeof(float));
    off[5] = o;
    o += align256(kla::diag_fwd_workspace(B, T, H, Dk, Dv));
    off[6] = o;
    return o;
}

size_t bwd_ws_layout(int B, int T, int H, int Dk, int Dv, bool have_S_chunks, size_t* off) {
    const size_t NC = (size_t)(T + kla::kChunkLen - 1) / kla::kChunkLen;
    const size_t ntok = (size_t)B * T * H;
    size_t o = 0;
    off[0] = o;  // S_chunks
    if (!have_S_chunks) o += align256((size_t)B * H * NC * Dk * Dv * sizeof(float));
    off[1] = o;  // acc_dq
    o += align256(ntok * Dk * sizeof(float));
    off[2] = o;  // acc_dkh
    o += align256(ntok * Dk * sizeof(float));
    off[3] = o;  // acc_db, acc_dc, acc_dG (contiguous, zeroed together with the above)
    o += align256(3 * ntok * sizeof(float));
    off[4] = o;
    return o;
}

}  // namespace

namespace kla {
int set_last_error(int status, const char* msg) {
    g_last_error = msg;
    return status;
}
}  // namespace kla

extern "C" {

const char* kla_status_string(int status) {
    switch (status) {
        case KLA_OK: return "KLA_OK";
        case KLA_ERR_INVALID_ARG: return "KLA_ERR_INVALID_ARG";
        case KLA_ERR_UNSUPPORTED: return "KLA_ERR_UNSUPPORTED";
        case KLA_ERR_WORKSPACE: return "KLA_ERR_WORKSPACE";
        case KLA_ERR_CUDA: return "KLA_ERR_CUDA";
        case KLA_ERR_TIMEOUT: return "KLA_ERR_TIMEOUT";
        default: return "KLA_ERR_UNKNOWN";
    }
}

const char* kla_last_error(void) { return g_last_error.c_str(); }

int kla_version(void) { return 100; }

size_t kla_chunk_fwd_workspace(int B, int T, int H, int Dk, int Dv, int chunk, int dtype) {
    take_beta_flag(dtype);
    if (B < 1 || H < 1 || T < 1 || chunk != kla::kChunkLen) return 0;
    kla::FwdArgs a{};
    a.B = B; a.T = T; a.H = H; a.Dk = Dk; a.Dv = Dv; a.bf16 = dtype == KLA_BF16;
    return kla::chunk_fwd_split_workspace(a);
}

int kla_chunk_fwd_kernel_launches(int B, int T, int H, int Dk, int Dv, int chunk, int dtype) {
    take_beta_flag(dtype);
    if (B < 1 || H < 1 || T < 1 || chunk != kla::kChunkLen) return 0;
    kla::FwdArgs a{};
    a.B = B; a.T = T; a.H = H; a.Dk = Dk; a.Dv = Dv; a.bf16 = dtype == KLA_BF16;
    return kla::chunk_fwd_split_workspace(a) > 0 ? kla::chunk_fwd_split_launches(a) : 1;
}

kla_status kla_chunk_fwd(const void* q, const void* k, const void* v, const float* eta,
                         const float* g, float eps, const float* S0, void* o, float* S_T,
                         float* S_chunks, int B, int T, int H, int Dk, int Dv, int chunk,
                         int dtype, int out_dtype, void* ws, size_t ws_bytes, void* stream) {
    const bool direct = take_beta_flag(dtype);
    kla_status st = check_common(B, T, H, Dk, Dv, chunk, dtype, out_dtype, eps);
    if (st != KLA_OK) return st;
    if (T > 0) {
        REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(eta); REQUIRE_PTR(g);
    }
    OPTIONAL_PTR(S0); OPTIONAL_PTR(o); OPTIONAL_PTR(S_T); OPTIONAL_PTR(S_chunks);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (S_T != nullptr && S_T != S0) {
            const size_t bytes = (size_t)B * H * Dk * Dv * sizeof(float);
            cudaError_t e = S0 ? cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s)
                               : cudaMemsetAsync(S_T, 0, bytes, s);
            if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_fwd(T=0)");
        }
        return KLA_OK;
    }
    kla::FwdArgs a{q, k, v, eta, g, kernel_eps(eps, direct), S0, o, S_T, S_chunks, B, T, H, Dk, Dv,
                   dtype == KLA_BF16, out_dtype == KLA_BF16};
    cudaError_t e;
    if (kla::chunk_fwd_tc_supported(a)) {
        // With the workspace of kla_chunk_fwd_workspace: chunk-parallel preparation + state pass
        // (segmented for long sequences over few heads).  Without it: the fused one-kernel path.
        const size_t need = kla::chunk_fwd_split_workspace(a);
        if (need > 0 && ws != nullptr && ws_bytes >= need) {
            if (!aligned32(ws)) return fail(KLA_ERR_INVALID_ARG, "ws must be 32-byte aligned");
            e = kla::launch_chunk_fwd_split(a, ws, s);
        } else {
            e = kla::launch_chunk_fwd_tc(a, s);
        }
    } else {
        e = kla::launch_chunk_fwd_simt(a, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_fwd launch");
    return KLA_OK;
}

static kla_status split_stage_checks(int B, int T, int H, int Dk, int Dv, int chunk, int dtype, int out_dtype,
                                     float eps, void* ws, size_t ws_bytes, const char* name, kla::FwdArgs* a) {
    kla_status st = check_common(B, T, H, Dk, Dv, chunk, dtype, out_dtype, eps);
    if (st != KLA_OK) return st;
    if (T < 1) return fail(KLA_ERR_INVALID_ARG, "%s needs T >= 1 (got %d)", name, T);
    a->B = B; a->T = T; a->H = H; a->Dk = Dk; a->Dv = Dv; a->eps = eps;
    a->bf16 = dtype == KLA_BF16; a->out_bf16 = out_dtype == KLA_BF16;
    if (!(a->bf16 && Dk == 128 && Dv == 128))
        return fail(KLA_ERR_UNSUPPORTED, "%s needs bf16 inputs with Dk == Dv == 128", name);
    const size_t need = kla::chunk_fwd_split_workspace(*a);
    if (ws == nullptr || ws_bytes < need)
        return fail(KLA_ERR_WORKSPACE, "%s needs %zu workspace bytes (got %zu)", name, need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    if (!aligned32(ws)) return fail(KLA_ERR_INVALID_ARG, "ws must be 32-byte aligned");
    return KLA_OK;
}

kla_status kla_chunk_fwd_prep(const void* q, const void* k, const void* v, const float* eta,
                              const float* g, float eps, int B, int T, int H, int Dk, int Dv,
                              int chunk, int dtype, void* ws, size_t ws_bytes, void* stream) {
    const bool direct = take_beta_flag(dtype);
    kla::FwdArgs a{};
    kla_status st = split_stage_checks(B, T, H, Dk, Dv, chunk, dtype, KLA_F32, eps, ws, ws_bytes,
                                       "kla_chunk_fwd_prep", &a);
    if (st != KLA_OK) return st;
    a.eps = kernel_eps(eps, direct);
    REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(eta); REQUIRE_PTR(g);
    a.q = q; a.k = k; a.v = v; a.eta = eta; a.g = g;
    cudaError_t e = kla::launch_chunk_fwd_split_prep(a, ws, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_fwd_prep launch");
    return KLA_OK;
}

kla_status kla_chunk_fwd_state_stage(int stage, const void* q, const void* v, const float* g, const float* S0,
                                     void* o, float* S_T, float* S_chunks, int B, int T, int H, int Dk, int Dv,
                                     int chunk, int dtype, int out_dtype, void* ws, size_t ws_bytes, void* stream) {
    take_beta_flag(dtype);  // the state pass reads the preparation's coefficients
    if (stage < 0 || stage > 3) return fail(KLA_ERR_INVALID_ARG, "stage must be 0, 1, 2 or 3 (got %d)", stage);
    kla::FwdArgs a{};
    kla_status st = split_stage_checks(B, T, H, Dk, Dv, chunk, dtype, out_dtype, 0.f, ws, ws_bytes,
                                       "kla_chunk_fwd_state", &a);
    if (st != KLA_OK) return st;
    REQUIRE_PTR(q); REQUIRE_PTR(v); REQUIRE_PTR(g);
    OPTIONAL_PTR(S0); OPTIONAL_PTR(o); OPTIONAL_PTR(S_T); OPTIONAL_PTR(S_chunks);
    a.q = q; a.v = v; a.g = g; a.S0 = S0; a.o = o; a.S_T = S_T; a.S_chunks = S_chunks;
    cudaError_t e = kla::launch_chunk_fwd_split_state(a, ws, static_cast<cudaStream_t>(stream), stage);
    if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_fwd_state launch");
    return KLA_OK;
}

kla_status kla_chunk_fwd_state(const void* q, const void* v, const float* g, const float* S0, void* o,
                               float* S_T, float* S_chunks, int B, int T, int H, int Dk, int Dv, int chunk,
                               int dtype, int out_dtype, void* ws, size_t ws_bytes, void* stream) {
    return kla_chunk_fwd_state_stage(0, q, v, g, S0, o, S_T, S_chunks, B, T, H, Dk, Dv, chunk, dtype, out_dtype, ws,
                                     ws_bytes, stream);
}

int kla_chunk_fwd_state_segments(int B, int T, int H, int Dk, int Dv, int chunk, int dtype) {
    take_beta_flag(dtype);
    kla::FwdArgs a{};
    if (B < 1 || H < 1 || T < 1 || chunk != kla::kChunkLen || dtype != KLA_BF16 || Dk != 128 || Dv != 128) return 0;
    a.B = B; a.T = T; a.H = H; a.Dk = Dk; a.Dv = Dv; a.bf16 = true;
    return kla::chunk_fwd_split_segments(a);
}

size_t kla_chunk_bwd_workspace_min(int B, int T, int H, int Dk, int Dv, int chunk, int dtype,
                                   int have_S_chunks) {
    (void)chunk;
    take_beta_flag(dtype);
    if (B < 1 || H < 1 || T < 0) return 0;
    size_t off[5];
    return bwd_ws_layout(B, T, H, Dk, Dv, have_S_chunks != 0, off);
}

int kla_chunk_bwd_reverse_segments(int B, int T, int H, int Dk, int Dv, int chunk, int dtype) {
    take_beta_flag(dtype);
    if (B < 1 || H < 1 || T < 1 || chunk != kla::kChunkLen || !tc_bwd_shape(T, Dk, Dv, dtype)) return 0;
    const int NC = (T + kla::kChunkLen - 1) / kla::kChunkLen;
    const int ns = kla::reverse_nseg(B * H, NC);
    if (ns <= 1) return 1;
    const int segc = (NC + ns - 1) / ns;
    return (NC + segc - 1) / segc;
}

int kla_chunk_bwd_reverse_slab_chunks(int B, int T, int H, int Dk, int Dv, int chunk, int dtype) {
    take_beta_flag(dtype);
    if (B < 1 || H < 1 || T < 1 || chunk != kla::kChunkLen || !tc_bwd_shape(T, Dk, Dv, dtype)) return 0;
    const int NC = (T + kla::kChunkLen - 1) / kla::kChunkLen;
    if (kla::reverse_nseg(B * H, NC) > 1) return 0;
    return kla::bwd_slab_newest(B * H, NC);
}

size_t kla_chunk_bwd_workspace(int B, int T, int H, int Dk, int Dv, int chunk, int dtype,
                               int have_S_chunks) {
    take_beta_flag(dtype);
    const size_t simt = kla_chunk_bwd_workspace_min(B, T, H, Dk, Dv, chunk, dtype, have_S_chunks);
    if (!tc_bwd_shape(T, Dk, Dv, dtype)) return simt;
    const size_t tc = kla::chunk_bwd_tc_workspace(B, T, H, have_S_chunks != 0);
    return tc > simt ? tc : simt;
}

}  // extern "C"

namespace {

// Backward of every entry point.  after_train: ws holds what kla_chunk_fwd_train left there for
// these inputs (the forward is not recomputed, S_chunks is ignored).
kla_status bwd_impl(const void* q, const void* k, const void* v, const float* eta, const float* g,
                    float eps, const float* S0, const void* dO, const float* dS_T, const float* S_chunks,
                    void* dq, void* dk, void* dv, float* deta, float* dg, float* dS0, int B, int T, int H,
                    int Dk, int Dv, int chunk, int dtype, int out_dtype, void* ws, size_t ws_bytes,
                    void* stream, bool after_train, const char* name) {
    const bool direct = take_beta_flag(dtype);
    kla_status st = check_common(B, T, H, Dk, Dv, chunk, dtype, out_dtype, eps);
    const float keps = kernel_eps(eps, direct);
    if (st != KLA_OK) return st;
    REQUIRE_PTR(dS0);
    OPTIONAL_PTR(S0); OPTIONAL_PTR(dS_T); OPTIONAL_PTR(S_chunks);
    if (after_train) S_chunks = nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t sbytes = (size_t)B * H * Dk * Dv * sizeof(float);
    if (T == 0) {
        cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, sbytes, cudaMemcpyDeviceToDevice, s)
                             : cudaMemsetAsync(dS0, 0, sbytes, s);
        if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_bwd(T=0)");
        return KLA_OK;
    }
    REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(eta); REQUIRE_PTR(g);
    REQUIRE_PTR(dO); REQUIRE_PTR(dq); REQUIRE_PTR(dk); REQUIRE_PTR(dv); REQUIRE_PTR(deta);
    REQUIRE_PTR(dg);
    size_t off[5];
    const size_t need = bwd_ws_layout(B, T, H, Dk, Dv, S_chunks != nullptr, off);
    if (ws == nullptr || ws_bytes < need)
        return fail(KLA_ERR_WORKSPACE, "%s needs %zu workspace bytes (got %zu)", name, need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    if (!aligned32(ws)) return fail(KLA_ERR_INVALID_ARG, "ws must be 32-byte aligned");
    cudaError_t e;
    if (tc_bwd_path(B, T, H, Dk, Dv, dtype, ws_bytes)) {
        kla::BwdTcArgs ta{q, k, v, eta, g, keps, S0, dO, dS_T, S_chunks, dq, dk, dv, deta, dg, dS0,
                          B, T, H, out_dtype == KLA_BF16};
        e = after_train ? kla::launch_chunk_bwd_tc_reverse(ta, ws, ws_bytes, s)
                        : kla::launch_chunk_bwd_tc(ta, ws, ws_bytes, s);
        if (e != cudaSuccess) return cuda_fail(e, name);
        return KLA_OK;
    }
    char* w = static_cast<char*>(ws);
    e = cudaMemsetAsync(w + off[1], 0, off[4] - off[1], s);
    if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_bwd workspace clear");
    const float* Sc = S_chunks;
    if (Sc == nullptr) {
        float* Sc_ws = reinterpret_cast<float*>(w + off[0]);
        if (!after_train) {
            kla::FwdArgs fa{q, k, v, eta, g, keps, S0, nullptr, nullptr, Sc_ws, B, T, H, Dk, Dv,
                            dtype == KLA_BF16, false};
            e = kla::chunk_fwd_tc_supported(fa) ? kla::launch_chunk_fwd_tc(fa, s) : kla::launch_chunk_fwd_simt(fa, s);
            if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_bwd state recompute");
        }
        Sc = Sc_ws;
    }
    const size_t ntok = (size_t)B * T * H;
    float* acc3 = reinterpret_cast<float*>(w + off[3]);
    kla::BwdArgs a{q, k, v, eta, g, keps, Sc, dO, dS_T, dq, dk, dv, deta, dg, dS0,
                   reinterpret_cast<float*>(w + off[1]), reinterpret_cast<float*>(w + off[2]),
                   acc3, acc3 + ntok, acc3 + 2 * ntok, B, T, H, Dk, Dv, dtype == KLA_BF16,
                   out_dtype == KLA_BF16};
    e = kla::launch_chunk_bwd_simt(a, s);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return KLA_OK;
}

}  // namespace

extern "C" {

kla_status kla_chunk_bwd(const void* q, const void* k, const void* v, const float* eta,
                         const float* g, float eps, const float* S0, const void* dO,
                         const float* dS_T, const float* S_chunks, void* dq, void* dk, void* dv,
                         float* deta, float* dg, float* dS0, int B, int T, int H, int Dk, int Dv,
                         int chunk, int dtype, int out_dtype, void* ws, size_t ws_bytes, void* stream) {
    return bwd_impl(q, k, v, eta, g, eps, S0, dO, dS_T, S_chunks, dq, dk, dv, deta, dg, dS0, B, T, H, Dk, Dv,
                    chunk, dtype, out_dtype, ws, ws_bytes, stream, false, "kla_chunk_bwd");
}

kla_status kla_chunk_fwd_train(const void* q, const void* k, const void* v, const float* eta,
                               const float* g, float eps, const float* S0, void* o, float* S_T, int B,
                               int T, int H, int Dk, int Dv, int chunk, int dtype, int out_dtype, void* ws,
                               size_t ws_bytes, void* stream) {
    const bool direct = take_beta_flag(dtype);
    kla_status st = check_common(B, T, H, Dk, Dv, chunk, dtype, out_dtype, eps);
    if (st != KLA_OK) return st;
    if (T > 0) {
        REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(eta); REQUIRE_PTR(g);
    }
    OPTIONAL_PTR(S0); OPTIONAL_PTR(o); OPTIONAL_PTR(S_T);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0)  // nothing for the backward to keep: the plain forward's empty-sequence case
        return kla_chunk_fwd(q, k, v, eta, g, eps, S0, o, S_T, nullptr, B, T, H, Dk, Dv, chunk,
                             dtype | (direct ? KLA_BETA_DIRECT : 0), out_dtype, nullptr, 0, stream);
    size_t off[5];
    const size_t need = bwd_ws_layout(B, T, H, Dk, Dv, false, off);
    if (ws == nullptr || ws_bytes < need)
        return fail(KLA_ERR_WORKSPACE, "kla_chunk_fwd_train needs %zu workspace bytes (got %zu)", need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    if (!aligned32(ws)) return fail(KLA_ERR_INVALID_ARG, "ws must be 32-byte aligned");
    kla::FwdArgs a{q, k, v, eta, g, kernel_eps(eps, direct), S0, o, S_T, nullptr, B, T, H, Dk, Dv,
                   dtype == KLA_BF16, out_dtype == KLA_BF16};
    cudaError_t e;
    if (tc_bwd_path(B, T, H, Dk, Dv, dtype, ws_bytes)) {
        e = kla::launch_chunk_fwd_train_tc(a, ws, ws_bytes, s);
    } else {
        // the CUDA-core backward's layout: the chunk states at the start of ws
        a.S_chunks = reinterpret_cast<float*>(static_cast<char*>(ws) + off[0]);
        e = kla::chunk_fwd_tc_supported(a) ? kla::launch_chunk_fwd_tc(a, s) : kla::launch_chunk_fwd_simt(a, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_fwd_train launch");
    return KLA_OK;
}

kla_status kla_chunk_bwd_after_train(const void* q, const void* k, const void* v, const float* eta,
                                     const float* g, float eps, const void* dO, const float* dS_T, void* dq,
                                     void* dk, void* dv, float* deta, float* dg, float* dS0, int B, int T,
                                     int H, int Dk, int Dv, int chunk, int dtype, int out_dtype, void* ws,
                                     size_t ws_bytes, void* stream) {
    return bwd_impl(q, k, v, eta, g, eps, nullptr, dO, dS_T, nullptr, dq, dk, dv, deta, dg, dS0, B, T, H, Dk,
                    Dv, chunk, dtype, out_dtype, ws, ws_bytes, stream, true, "kla_chunk_bwd_after_train");
}

kla_status kla_decode_step(const void* q, const void* k, const void* v, const float* eta,
                           const float* g, float eps, float* S, void* o, int B, int H, int Dk,
                           int Dv, int dtype, int out_dtype, void* stream) {
    const bool direct = take_beta_flag(dtype);
    kla_status st = check_common(B, 0, H, Dk, Dv, kla::kChunkLen, dtype, out_dtype, eps);
    if (st != KLA_OK) return st;
    REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(eta); REQUIRE_PTR(g);
    REQUIRE_PTR(S);
    OPTIONAL_PTR(o);
    kla::DecodeArgs a{q, k, v, eta, g, kernel_eps(eps, direct), S, o, B, H, Dk, Dv, dtype == KLA_BF16,
                      out_dtype == KLA_BF16, g_inject_timeout.exchange(0) != 0};
    cudaError_t e = kla::launch_decode(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kla_decode_step launch");
    return KLA_OK;
}

kla_status kla_decode_step_diag(const void* q, const void* k, const void* v, const float* eta,
                                const float* g, float eps, float* S, void* o, int B, int H, int Dk,
                                int Dv, int dtype, int out_dtype, void* stream) {
    const bool direct = take_beta_flag(dtype);
    kla_status st = check_common(B, 0, H, Dk, Dv, kla::kChunkLen, dtype, out_dtype, eps);
    if (st != KLA_OK) return st;
    REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(eta); REQUIRE_PTR(g);
    REQUIRE_PTR(S);
    OPTIONAL_PTR(o);
    kla::DecodeArgs a{q, k, v, eta, g, kernel_eps(eps, direct), S, o, B, H, Dk, Dv, dtype == KLA_BF16,
                      out_dtype == KLA_BF16, false, true};
    cudaError_t e = kla::launch_decode(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kla_decode_step_diag launch");
    return KLA_OK;
}

namespace {
// FwdArgs of a diagonal-gated forward with only the sizes and types set (workspace queries).
kla::FwdArgs diag_shape(int B, int T, int H, int Dk, int Dv, int dtype) {
    kla::FwdArgs a{};
    a.B = B;
    a.T = T;
    a.H = H;
    a.Dk = Dk;
    a.Dv = Dv;
    a.bf16 = dtype == KLA_BF16;
    a.diag = true;
    return a;
}
}  // namespace

size_t kla_chunk_fwd_diag_workspace(int B, int T, int H, int Dk, int Dv, int chunk, int dtype) {
    take_beta_flag(dtype);
    if (B < 1 || H < 1 || T < 1 || chunk != kla::kChunkLen || (Dk != 64 && Dk != 128) || (Dv != 64 && Dv != 128))
        return 0;
    const kla::FwdArgs a = diag_shape(B, T, H, Dk, Dv, dtype);
    if (kla::chunk_fwd_diag_tc_supported(a)) return kla::chunk_fwd_split_workspace(a);
    return kla::diag_fwd_workspace(B, T, H, Dk, Dv);
}

int kla_chunk_fwd_diag_kernel_launches(int B, int T, int H, int Dk, int Dv, int chunk, int dtype) {
    take_beta_flag(dtype);
    if (B < 1 || H < 1 || T < 1 || chunk != kla::kChunkLen || (Dk != 64 && Dk != 128) || (Dv != 64 && Dv != 128))
        return 0;
    const kla::FwdArgs a = diag_shape(B, T, H, Dk, Dv, dtype);
    return kla::chunk_fwd_diag_tc_supported(a) ? kla::chunk_fwd_split_launches(a) : 2;
}

kla_status kla_chunk_fwd_diag(const void* q, const void* k, const void* v, const float* eta,
                              const float* g, float eps, const float* S0, void* o, float* S_T, int B,
                              int T, int H, int Dk, int Dv, int chunk, int dtype, int out_dtype,
                              void* ws, size_t ws_bytes, void* stream) {
    const bool direct = take_beta_flag(dtype);
    kla_status st = check_common(B, T, H, Dk, Dv, chunk, dtype, out_dtype, eps);
    if (st != KLA_OK) return st;
    if (T > 0) {
        REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(eta); REQUIRE_PTR(g);
    }
    OPTIONAL_PTR(S0); OPTIONAL_PTR(o); OPTIONAL_PTR(S_T);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (S_T != nullptr && S_T != S0) {
            const size_t bytes = (size_t)B * H * Dk * Dv * sizeof(float);
            cudaError_t e = S0 ? cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s)
                               : cudaMemsetAsync(S_T, 0, bytes, s);
            if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_fwd_diag(T=0)");
        }
        return KLA_OK;
    }
    if (!aligned32(ws)) return fail(KLA_ERR_INVALID_ARG, "ws must be 32-byte aligned");
    kla::FwdArgs a{q, k, v, eta, g, kernel_eps(eps, direct), S0, o, S_T, nullptr, B, T, H, Dk, Dv,
                   dtype == KLA_BF16, out_dtype == KLA_BF16};
    a.diag = true;
    cudaError_t e;
    if (kla::chunk_fwd_diag_tc_supported(a) && ws != nullptr && ws_bytes >= kla::chunk_fwd_split_workspace(a)) {
        // bf16, Dk = Dv = 128: preparation and state pass on the tensor cores (64-token chunks)
        e = kla::launch_chunk_fwd_split(a, ws, s);
    } else {
        // CUDA cores, 16-token chunks: split with a large enough workspace, else one kernel
        a.diag = false;
        e = kla::launch_chunk_fwd_diag(a, ws, ws == nullptr ? 0 : ws_bytes, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_fwd_diag launch");
    return KLA_OK;
}

size_t kla_chunk_bwd_diag_workspace(int B, int T, int H, int Dk, int Dv, int chunk, int dtype) {
    (void)chunk;
    take_beta_flag(dtype);
    if (B < 1 || H < 1 || T < 0) return 0;
    size_t off[7];
    return diag_bwd_ws_layout(B, T, H, Dk, Dv, off);
}

kla_status kla_chunk_bwd_diag(const void* q, const void* k, const void* v, const float* eta,
                              const float* g, float eps, const float* S0, const void* dO,
                              const float* dS_T, void* dq, void* dk, void* dv, float* deta, float* dg,
                              float* dS0, int B, int T, int H, int Dk, int Dv, int chunk, int dtype,
                              int out_dtype, void* ws, size_t ws_bytes, void* stream) {
    const bool direct = take_beta_flag(dtype);
    kla_status st = check_common(B, T, H, Dk, Dv, chunk, dtype, out_dtype, eps);
    if (st != KLA_OK) return st;
    REQUIRE_PTR(dS0);
    OPTIONAL_PTR(S0); OPTIONAL_PTR(dS_T);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        const size_t sbytes = (size_t)B * H * Dk * Dv * sizeof(float);
        cudaError_t e = dS_T ? cudaMemcpyAsync(dS0, dS_T, sbytes, cudaMemcpyDeviceToDevice, s)
                             : cudaMemsetAsync(dS0, 0, sbytes, s);
        if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_bwd_diag(T=0)");
        return KLA_OK;
    }
    REQUIRE_PTR(q); REQUIRE_PTR(k); REQUIRE_PTR(v); REQUIRE_PTR(eta); REQUIRE_PTR(g);
    REQUIRE_PTR(dO); REQUIRE_PTR(dq); REQUIRE_PTR(dk); REQUIRE_PTR(dv); REQUIRE_PTR(deta);
    REQUIRE_PTR(dg);
    size_t off[7];
    const size_t need = diag_bwd_ws_layout(B, T, H, Dk, Dv, off);
    if (ws == nullptr || ws_bytes < need)
        return fail(KLA_ERR_WORKSPACE, "kla_chunk_bwd_diag needs %zu workspace bytes (got %zu)", need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    if (!aligned32(ws)) return fail(KLA_ERR_INVALID_ARG, "ws must be 32-byte aligned");
    char* w = static_cast<char*>(ws);
    cudaError_t e = cudaMemsetAsync(w + off[1], 0, off[5] - off[1], s);
    if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_bwd_diag workspace clear");
    const size_t ntok = (size_t)B * T * H;
    float* acc_b = reinterpret_cast<float*>(w + off[4]);
    kla::BwdArgs a{q, k, v, eta, g, kernel_eps(eps, direct), reinterpret_cast<const float*>(w + off[0]), dO, dS_T,
                   dq, dk, dv, deta, dg, dS0, reinterpret_cast<float*>(w + off[1]),
                   reinterpret_cast<float*>(w + off[2]), acc_b, acc_b + ntok,
                   reinterpret_cast<float*>(w + off[3]), B, T, H, Dk, Dv, dtype == KLA_BF16,
                   out_dtype == KLA_BF16};
    e = kla::launch_chunk_bwd_diag(a, S0, w + off[5], need - off[5], s);
    if (e != cudaSuccess) return cuda_fail(e, "kla_chunk_bwd_diag launch");
    return KLA_OK;
}

static kla_status gate_checks(int N, int D, int H, int Dk, int dtype, bool with_q) {
    if (N < 0 || D < 1 || H < 1)
        return fail(KLA_ERR_INVALID_ARG, "sizes must satisfy N>=0, D>=1, H>=1 (got N=%d D=%d H=%d)", N, D, H);
    if (H > 64) return fail(KLA_ERR_UNSUPPORTED, "at most 64 heads (got H=%d)", H);
    if (dtype != KLA_F32 && dtype != KLA_BF16)
        return fail(KLA_ERR_UNSUPPORTED, "dtype must be KLA_F32 or KLA_BF16 (got %d)", dtype);
    if (D % 8 != 0) return fail(KLA_ERR_UNSUPPORTED, "D must be a multiple of 8 (got D=%d)", D);
    if (with_q && Dk != 64 && Dk != 128) return fail(KLA_ERR_UNSUPPORTED, "Dk must be 64 or 128 (got %d)", Dk);
    return KLA_OK;
}

kla_status kla_gate_prologue(const void* x, const void* W, const float* bias, const void* q, float* eta, float* g,
                             void* q_hat, int N, int D, int H, int Dk, int dtype, void* stream) {
    if ((q == nullptr) != (q_hat == nullptr))
        return fail(KLA_ERR_INVALID_ARG, "q and q_hat must be given together (or both NULL)");
    kla_status st = gate_checks(N, D, H, Dk, dtype, q != nullptr);
    if (st != KLA_OK) return st;
    if (N == 0) return KLA_OK;
    REQUIRE_PTR(x); REQUIRE_PTR(W); REQUIRE_PTR(bias); REQUIRE_PTR(eta); REQUIRE_PTR(g);
    OPTIONAL_PTR(q); OPTIONAL_PTR(q_hat);
    kla::GateArgs a{x, W, bias, q, eta, g, q_hat, N, D, H, Dk, dtype == KLA_BF16};
    cudaError_t e = kla::launch_gate_prologue(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kla_gate_prologue launch");
    return KLA_OK;
}

size_t kla_gate_prologue_bwd_workspace(int N, int D, int H) {
    if (N < 0 || D < 1 || H < 1) return 0;
    return kla::gate_bwd_workspace(N, D, H);
}

kla_status kla_gate_prologue_bwd(const void* x, const void* W, const float* eta, const float* g, const void* q,
                                 const float* deta, const float* dg, const float* dq_hat, float* dx, float* dW,
                                 float* dbias, float* dq, int N, int D, int H, int Dk, int dtype, void* ws,
                                 size_t ws_bytes, void* stream) {
    if ((q == nullptr) != (dq_hat == nullptr) || (q == nullptr) != (dq == nullptr))
        return fail(KLA_ERR_INVALID_ARG, "q, dq_hat and dq must be given together (or all NULL)");
    kla_status st = gate_checks(N, D, H, Dk, dtype, q != nullptr);
    if (st != KLA_OK) return st;
    REQUIRE_PTR(dW); REQUIRE_PTR(dbias);
    if (N > 0) {
        REQUIRE_PTR(x); REQUIRE_PTR(W); REQUIRE_PTR(eta); REQUIRE_PTR(g); REQUIRE_PTR(deta); REQUIRE_PTR(dg);
        REQUIRE_PTR(dx);
    }
    OPTIONAL_PTR(q); OPTIONAL_PTR(dq_hat); OPTIONAL_PTR(dq);
    const size_t need = kla::gate_bwd_workspace(N, D, H);
    if (N > 0 && (ws == nullptr || ws_bytes < need))
        return fail(KLA_ERR_WORKSPACE, "kla_gate_prologue_bwd needs %zu workspace bytes (got %zu)", need,
                    ws == nullptr ? (size_t)0 : ws_bytes);
    if (!aligned32(ws)) return fail(KLA_ERR_INVALID_ARG, "ws must be 32-byte aligned");
    kla::GateBwdArgs a{x, W, eta, g, deta, dg, q, dq_hat, dx, dW, dbias, dq, N, D, H, Dk, dtype == KLA_BF16};
    cudaError_t e = kla::launch_gate_prologue_bwd(a, ws, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kla_gate_prologue_bwd launch");
    return KLA_OK;
}

void kla_debug_inject_wait_timeout(void) { g_inject_timeout.store(1); }

kla_status kla_check_device_error(void* stream) {
    unsigned int flag = 0, flag2 = 0, flag3 = 0, flag4 = 0, flag5 = 0;
    cudaError_t e = kla::tc_take_error(static_cast<cudaStream_t>(stream), &flag);
    if (e == cudaSuccess) e = kla::decode_take_error(static_cast<cudaStream_t>(stream), &flag2);
    if (e == cudaSuccess) e = kla::split_take_error(static_cast<cudaStream_t>(stream), &flag3);
    if (e == cudaSuccess) e = kla::bwd_tc_take_error(static_cast<cudaStream_t>(stream), &flag4);
    if (e == cudaSuccess) e = kla::gates_take_error(static_cast<cudaStream_t>(stream), &flag5);
    unsigned int flag6 = 0;
    if (e == cudaSuccess) e = kla::diag_take_error(static_cast<cudaStream_t>(stream), &flag6);
    flag5 |= flag6 << 1;
    if (e != cudaSuccess) return cuda_fail(e, "kla_check_device_error");
    flag |= (flag2 << 8) | (flag3 << 16) | (flag4 << 24) | (flag5 << 4);
    if (flag) return fail(KLA_ERR_TIMEOUT, "a kernel gave up on a bounded wait (flag %u)", flag);
    return KLA_OK;
}

}  // extern "C"
