// Forward entry point for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the operator:
// code inside a framework's memory pool, or runtimes that forbid allocation on the
// hot path. gdn_chunk_fwd_noalloc runs the same forward as gdn_chunk_fwd but takes its
// scratch (the status word and, for packed sequences under context parallelism, the
// segment table) from a fixed array in the library's device memory instead of a
// caller workspace. The caller still provides every input and output buffer.
#include <cstdio>
#include <mutex>

#include "gdn_common.cuh"

namespace {

// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;   // 1 MiB
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device. The array's host-side name is not
// a device address, so it is looked up once per device (with that device current).
gdn_status scratch_address(void** out) {
  int dev = 0;
  const cudaError_t derr = cudaGetDevice(&dev);
  if (derr != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    char msg[160];
    if (derr != cudaSuccess)
      snprintf(msg, sizeof(msg), "gdn_chunk_fwd_noalloc: cudaGetDevice: %s", cudaGetErrorString(derr));
    else
      snprintf(msg, sizeof(msg), "gdn_chunk_fwd_noalloc: device index %d beyond the %d the library tracks", dev,
               kMaxDevices);
    gdn::set_last_error(msg);
    return GDN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess || p == nullptr) {
      char msg[160];
      snprintf(msg, sizeof(msg), "no-alloc scratch address lookup: %s", cudaGetErrorString(err));
      gdn::set_last_error(msg);
      return GDN_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return GDN_OK;
}

}  // namespace

extern "C" gdn_status gdn_chunk_fwd_noalloc(gdn_dtype dtype, int B, int T, int Hqk, int Hv, int dk, int dv,
                                             const void* q, const void* k, const void* v, const float* g,
                                             const void* beta, float scale, const float* h0,
                                             const int32_t* cu_seqlens, int num_seqs, void* o, float* hT,
                                             const gdn_options* opt, cudaStream_t stream) {
  gdn_options op{};
  if (opt) op = *opt;
  size_t need = gdn_chunk_fwd_workspace_size(B, T, Hqk, Hv, dk, dv, cu_seqlens ? num_seqs : 0, &op);
  if (need > kNoAllocScratchBytes && op.cp_exact == 2) {
    // the exact fallback of the gate-driven start keeps per-segment maps; with too little room, the
    // other fallback (restart at the sequence start) needs only the segment table
    op.cp_exact = 0;
    need = gdn_chunk_fwd_workspace_size(B, T, Hqk, Hv, dk, dv, cu_seqlens ? num_seqs : 0, &op);
  }
  if (need > kNoAllocScratchBytes) {                             // beyond the fixed array
    char msg[160];
    snprintf(msg, sizeof(msg), "gdn_chunk_fwd_noalloc: needs %zu bytes of scratch, the static array holds %zu",
             need, kNoAllocScratchBytes);
    gdn::set_last_error(msg);
    return GDN_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  gdn_status st = scratch_address(&scratch);
  if (st != GDN_OK) return st;
  // the status word must start at zero; the rest of the scratch is rewritten by every call
  const cudaError_t merr = cudaMemsetAsync(scratch, 0, gdn::kStatusBytes, stream);
  if (merr != cudaSuccess) {
    char msg[160];
    snprintf(msg, sizeof(msg), "gdn_chunk_fwd_noalloc: clearing the status word: %s", cudaGetErrorString(merr));
    gdn::set_last_error(msg);
    return GDN_ERR_CUDA;
  }
  return gdn_chunk_fwd(dtype, B, T, Hqk, Hv, dk, dv, q, k, v, g, beta, scale, h0, cu_seqlens, num_seqs, o, hT,
                       scratch, kNoAllocScratchBytes, &op, stream);
}
