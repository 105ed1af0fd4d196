// kla_bwd_noalloc.cu -- the backward pass for callers that cannot allocate device memory.
//
// kla_chunk_bwd needs a scratch workspace that the caller allocates.  Some callers cannot
// call cudaMalloc at all: code running inside a CUDA-graph capture that must not allocate,
// plugins of a host framework whose allocator is closed to them, or real-time paths where
// an allocation could block.  kla_chunk_bwd_noalloc serves them from a fixed scratch array
// compiled into this library instead.  It allocates nothing: no cudaMalloc, cudaFree or
// allocating library routine is called; the caller still passes every input and output.
#include <stdio.h>

#include <mutex>

#include "kla.h"
#include "kla_launch.h"

namespace {

// Fixed scratch in device global memory.  Every GPU that loads libkla.so holds these bytes
// until the process exits; all calls on a device share them.
constexpr size_t kNoallocScratchBytes = KLA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_bwd_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the symbol
// g_bwd_scratch is only a host-side handle, never a device address, so the address is
// looked up once per device (with that device current) and cached.
kla_status scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_bwd_scratch);
        if (e != cudaSuccess || p == nullptr) return KLA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KLA_OK;
}

}  // namespace

extern "C" {

size_t kla_chunk_bwd_noalloc_scratch_bytes(void) { return kNoallocScratchBytes; }

kla_status kla_chunk_bwd_noalloc(const void* q, const void* k, const void* v, const float* eta,
                                 const float* g, float eps, const float* S0, const void* dO,
                                 const float* dS_T, const float* S_chunks, void* dq, void* dk, void* dv,
                                 float* deta, float* dg, float* dS0, int B, int T, int H, int Dk, int Dv,
                                 int chunk, int dtype, int out_dtype, void* stream) {
    // Size check first, before touching the device: the scratch replaces the workspace.  The
    // bound is the CUDA-core backward's size; kla_chunk_bwd picks the tensor cores by itself
    // when their larger layout also fits the scratch.
    const size_t need = kla_chunk_bwd_workspace_min(B, T, H, Dk, Dv, chunk, dtype, S_chunks != nullptr);
    if (need > kNoallocScratchBytes) {
        // The regular entry point reports the same condition with its own message; run its
        // validation so argument errors keep their usual status, then report the size.
        kla_status st = kla_chunk_bwd(q, k, v, eta, g, eps, S0, dO, dS_T, S_chunks, dq, dk, dv, deta,
                                      dg, dS0, B, T, H, Dk, Dv, chunk, dtype, out_dtype, nullptr, 0, stream);
        if (st != KLA_ERR_WORKSPACE) return st;
        char msg[200];
        snprintf(msg, sizeof(msg),
                 "kla_chunk_bwd_noalloc: this call needs %zu scratch bytes, more than the %zu-byte "
                 "static scratch; use kla_chunk_bwd with a caller workspace",
                 need, kNoallocScratchBytes);
        return static_cast<kla_status>(kla::set_last_error(KLA_ERR_WORKSPACE, msg));
    }
    void* ws = nullptr;
    kla_status st = scratch_address(&ws);
    if (st != KLA_OK)
        return static_cast<kla_status>(
            kla::set_last_error(st, "kla_chunk_bwd_noalloc: could not resolve the scratch address"));
    return kla_chunk_bwd(q, k, v, eta, g, eps, S0, dO, dS_T, S_chunks, dq, dk, dv, deta, dg, dS0, B, T, H,
                         Dk, Dv, chunk, dtype, out_dtype, ws, kNoallocScratchBytes, stream);
}

}  // extern "C"
