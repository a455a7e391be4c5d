// Shared host/device definitions of the GDN chunked-prefill library.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "gdn.h"

namespace gdn {

constexpr int kChunk = 64;             // tokens per chunk
constexpr size_t kStatusBytes = 256;   // head of every workspace: device status word + padding

// Device-side error codes written into the workspace status word (first error wins).
enum DeviceError : int {
  kDevOk = 0,
  kDevTimeout = 1,       // a bounded mbarrier wait gave up
  kDevBadSeqlens = 2,    // cu_seqlens not monotone / not ending at T
  kDevMisaligned = 3,    // dynamic shared memory not at the 1024-byte alignment the swizzled tiles need
};

// Everything a forward kernel needs. Pointers are device pointers.
struct FwdParams {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const void* beta;
  const float* h0;          // nullable, [N,Hv,dk,dv]
  const int32_t* cu;        // nullable, [N+1]
  void* o;                  // nullable (no output written)
  float* hT;                // nullable
  int* status;              // device status word (head of the caller's workspace)
  int* status_dev;          // nullable: the library's per-device status word (gdn_check_device_error)
  int qk_l2norm;            // q, k rows divided by sqrt(|x|^2 + eps) inside the kernels
  int test_stall;           // testing only: the tensor-core forward's CTAs wait once on a barrier nothing completes
  // backward support: bf16 start state S (dv x dk, row-major) of every chunk, at
  // states + ((chunk_off[n] + chunk) * Hv + j) * dv * dk; chunk_off nullable -> n * ceil(T/64)
  __nv_bfloat16* states;    // nullable
  const int* chunk_off;     // nullable
  // backward support: A = (I + L)^-1 (fp32, 64 x 64 row-major) of every chunk, written by the
  // forward pass (state-store mode) at chunk_a + (slot * Hv + j) * 4096 (slot as for states); nullable
  float* chunk_a;
  // backward support: P = lower_incl(Q K^T * E) (bf16, the 8 KB 128B-swizzled tile of the
  // tensor-core operand) of every chunk, written by the forward pass, at
  // chunk_p + (slot * Hv + j) * 8192 bytes; nullable
  uint8_t* chunk_p;
  int B, T, Hqk, Hv, dk, dv, N;
  float scale;
};

__device__ __forceinline__ void record_error(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}
// Record a device-side finding in the call's workspace status word and in the library's
// per-device word (first error wins in each).
__device__ __forceinline__ void report_error(const FwdParams& p, int code) {
  record_error(p.status, code);
  record_error(p.status_dev, code);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ size_t chunk_slot(const FwdParams& p, int n, int chunk) {
  const int base = p.chunk_off ? p.chunk_off[n] : n * ((p.T + kChunk - 1) / kChunk);
  return (size_t)(base + chunk);
}

// Token span [s, e) and batch row of sequence n; returns false (after recording an
// error) when a packed cu_seqlens entry is out of range.
__device__ __forceinline__ bool seq_span(const FwdParams& p, int n, int& b, int& s, int& e) {
  if (p.cu == nullptr) {
    b = n; s = 0; e = p.T;
    return true;
  }
  b = 0;
  s = p.cu[n];
  e = p.cu[n + 1];
  if (s < 0 || e < s || e > p.T) {
    report_error(p, kDevBadSeqlens);
    return false;
  }
  if ((n == 0 && s != 0) || (n == p.N - 1 && e != p.T)) {
    report_error(p, kDevBadSeqlens);
    return false;
  }
  return true;
}

// ---- host-side launch instrumentation (gdn_api.cu)
enum KernelId : int { kKernFwdTc = 0, kKernFwdSimt = 1, kKernCpStitch = 2, kKernBwdTc = 3,
                      kKernBwdSimt = 4, kKernBwdReduce = 5, kKernCpPlan = 6, kKernBwdChain = 7,
                      kKernStep = 8, kKernCpProbe = 9, kKernCount = 10 };
void trace_pre(int kernel_id, cudaStream_t st);
void set_last_error(const char* msg);   // text returned by gdn_last_error() on this thread
void trace_post(cudaStream_t st);

}  // namespace gdn
