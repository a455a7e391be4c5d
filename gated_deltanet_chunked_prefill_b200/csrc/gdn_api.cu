// C-ABI entry points: argument validation, workspace layout, planning, launches.
#include <cstdio>
#include <cstring>

#include "gdn_common.cuh"
#include "gdn_tc.cuh"

namespace gdn {
cudaError_t launch_fwd_simt(const FwdParams& p, bool bf16, cudaStream_t st);
}

using namespace gdn;

namespace {

constexpr int kVersion = 100;  // 0.1.0

thread_local char g_last_error[256] = "";

gdn_status cuda_fail(const char* where, cudaError_t err) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(err), (int)err);
  return GDN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Shape {
  int B, T, Hqk, Hv, dk, dv, N;
  bool packed;
};

gdn_status check_shape(int B, int T, int Hqk, int Hv, int dk, int dv, int num_seqs, bool packed,
                       Shape& s) {
  if (B <= 0 || T < 0 || Hqk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return GDN_ERR_INVALID_ARG;
  if (Hv % Hqk != 0) return GDN_ERR_INVALID_ARG;
  if (packed && (B != 1 || num_seqs <= 0)) return GDN_ERR_INVALID_ARG;
  // element counts must fit the 32-bit token index arithmetic used for row offsets
  if ((long long)B * T * (long long)(Hv > Hqk ? Hv : Hqk) >= (1LL << 31)) return GDN_ERR_UNSUPPORTED;
  if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return GDN_ERR_UNSUPPORTED;
  s = Shape{B, T, Hqk, Hv, dk, dv, packed ? num_seqs : B, packed};
  return GDN_OK;
}


}  // namespace

extern "C" {

int gdn_version(void) { return kVersion; }

const char* gdn_last_error(void) { return g_last_error; }

const char* gdn_status_string(gdn_status s) {
  switch (s) {
    case GDN_OK: return "ok";
    case GDN_ERR_INVALID_ARG: return "invalid argument";
    case GDN_ERR_UNSUPPORTED: return "unsupported configuration";
    case GDN_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case GDN_ERR_CUDA: return "CUDA runtime error";
    case GDN_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait timed out";
    case GDN_ERR_DEVICE_INPUT: return "a kernel found inconsistent device input (cu_seqlens)";
  }
  return "unknown status";
}

size_t gdn_chunk_fwd_workspace_size(int B, int T, int Hqk, int Hv, int dk, int dv, int num_seqs,
                                    const gdn_options* opt) {
  (void)B; (void)T; (void)Hqk; (void)Hv; (void)dk; (void)dv; (void)num_seqs; (void)opt;
  return kStatusBytes;
}

gdn_status gdn_chunk_fwd(gdn_dtype dtype, int B, int T, int Hqk, int Hv, int dk, int dv,
                         const void* q, const void* k, const void* v, const float* g,
                         const void* beta, float scale, const float* h0, const int32_t* cu_seqlens,
                         int num_seqs, void* o, float* hT, void* workspace, size_t workspace_bytes,
                         const gdn_options* opt, cudaStream_t stream) {
  if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
  Shape s;
  gdn_status st = check_shape(B, T, Hqk, Hv, dk, dv, num_seqs, cu_seqlens != nullptr, s);
  if (st != GDN_OK) return st;
  if (opt) {
    for (int r : opt->reserved)
      if (r != 0) return GDN_ERR_INVALID_ARG;
  }
  if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, g, beta, h0, cu_seqlens, o, hT};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < gdn_chunk_fwd_workspace_size(B, T, Hqk, Hv, dk, dv, num_seqs, opt))
    return GDN_ERR_WORKSPACE;

  FwdParams p{};
  p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.h0 = h0; p.cu = cu_seqlens;
  p.o = o; p.hT = hT;
  p.status = static_cast<int*>(workspace);
  p.B = s.B; p.T = s.T; p.Hqk = s.Hqk; p.Hv = s.Hv; p.dk = s.dk; p.dv = s.dv; p.N = s.N;
  p.scale = scale;

  if (s.T == 0) return GDN_OK;
  cudaError_t err;
  if (dtype == GDN_BF16 && dk == 128 && dv == 128) {
    TcPlan plan{};
    plan.kind = kPlanUnits;
    const char* what = "";
    err = launch_fwd_tc(p, plan, s.N * s.Hv, stream, &what);
    if (err != cudaSuccess) return cuda_fail(what, err);
  } else {
    err = launch_fwd_simt(p, dtype == GDN_BF16, stream);
    if (err != cudaSuccess) return cuda_fail("CUDA-core forward", err);
  }
  return GDN_OK;
}

size_t gdn_chunk_bwd_workspace_size(int B, int T, int Hqk, int Hv, int dk, int dv, int num_seqs,
                                    const gdn_options* opt) {
  (void)B; (void)T; (void)Hqk; (void)Hv; (void)dk; (void)dv; (void)num_seqs; (void)opt;
  return kStatusBytes;
}

gdn_status gdn_chunk_bwd(gdn_dtype dtype, int B, int T, int Hqk, int Hv, int dk, int dv,
                         const void* q, const void* k, const void* v, const float* g,
                         const void* beta, float scale, const float* h0, const int32_t* cu_seqlens,
                         int num_seqs, const void* dO, const float* dhT, void* dq, void* dk_out,
                         void* dv_out, float* dg, void* dbeta, float* dh0, void* workspace,
                         size_t workspace_bytes, const gdn_options* opt, cudaStream_t stream) {
  (void)dtype; (void)B; (void)T; (void)Hqk; (void)Hv; (void)dk; (void)dv; (void)q; (void)k;
  (void)v; (void)g; (void)beta; (void)scale; (void)h0; (void)cu_seqlens; (void)num_seqs;
  (void)dO; (void)dhT; (void)dq; (void)dk_out; (void)dv_out; (void)dg; (void)dbeta; (void)dh0;
  (void)workspace; (void)workspace_bytes; (void)opt; (void)stream;
  return GDN_ERR_UNSUPPORTED;
}

gdn_status gdn_read_device_status(void* workspace, cudaStream_t stream) {
  if (!workspace) return GDN_ERR_WORKSPACE;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return GDN_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GDN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return GDN_ERR_CUDA;
  switch (code) {
    case kDevOk: return GDN_OK;
    case kDevTimeout: return GDN_ERR_DEVICE_TIMEOUT;
    default: return GDN_ERR_DEVICE_INPUT;
  }
}

}  // extern "C"
