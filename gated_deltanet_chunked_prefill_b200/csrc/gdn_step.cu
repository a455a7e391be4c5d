// One recurrent step of the gated delta rule per (sequence, v-head): the decode step that
// continues from a chunked prefill's final state. The pages list on-device agentic inference
// among the scenarios ("FlashQLA resource", section 4, table of the authors' stated results);
// generating after a prefill runs the recurrence one token at a time from hT.
//
// With h = S^T (dk x dv, fp32) the step is the token form of the recurrence:
//   h <- exp(g) h;   r = v - h^T k;   h <- h + beta k r^T;   o = scale h^T q.
// It moves the state once each way (2 dk dv fp32 per v-head) and does O(dk dv) flops, so it
// is HBM-bound. The dv columns of h are independent, so a CTA takes kCols of them for one
// (sequence, v-head): threads over those columns (rows of h are coalesced) and kRows thread
// rows over dk, with the two dot products over dk reduced through shared memory in a fixed
// order (bit-reproducible). Two CTAs fit on an SM, so one's loads overlap the other's
// reductions and stores.
#include <cstdio>

#include "gdn_common.cuh"

namespace gdn {
namespace {

// Columns of h per CTA (64, or 32 at dk = 256) and thread rows splitting dk (4, or 8 at dk = 256):
// 256 threads per CTA, each holding at most 32 entries of its column, two CTAs per SM.
template <int DK> constexpr int cols_for() { return DK == 256 ? 32 : 64; }
template <int DK> constexpr int rows_for() { return DK == 256 ? 8 : 4; }

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(cols_for<DK>() * rows_for<DK>(), 2)
gdn_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const float* __restrict__ g, const T* __restrict__ beta, float scale,
                float* __restrict__ state, T* __restrict__ o, int Hqk, int Hv) {
  constexpr int kRows = rows_for<DK>();
  constexpr int kCols = cols_for<DK>();
  constexpr int kPer = DK / kRows;            // dk entries of one column per thread
  __shared__ float ks[DK], qs[DK];
  constexpr int kSplit = DV / kCols;          // CTAs per (sequence, v-head)
  __shared__ float part_k[kRows][kCols], part_q[kRows][kCols];
  const int unit = blockIdx.x / kSplit;       // n * Hv + j
  const int j = unit % Hv, n = unit / Hv;
  const int hq = j / (Hv / Hqk);
  const int x = threadIdx.x, w = threadIdx.y;  // column slot x, row block w (dk)
  const int c = (blockIdx.x % kSplit) * kCols + x;   // column of h (dv)
  const int tid = w * kCols + x;
  const size_t qk_off = ((size_t)n * Hqk + hq) * DK;
  for (int d = tid; d < DK; d += kCols * kRows) {
    ks[d] = to_f(k[qk_off + d]);
    qs[d] = to_f(q[qk_off + d]);
  }
  __syncthreads();
  float* h = state + (size_t)unit * DK * DV + c;
  float hc[kPer];
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int d = w * kPer + i;
    hc[i] = h[(size_t)d * DV];
    acc = fmaf(hc[i], ks[d], acc);
  }
  part_k[w][x] = acc;
  __syncthreads();
  const float decay = expf(g[unit]);
  const float b = to_f(beta[unit]);
  float hk = 0.f;                             // (h^T k)_c of the old state, same order in every row
#pragma unroll
  for (int y = 0; y < kRows; ++y) hk += part_k[y][x];
  const float rc = to_f(v[(size_t)unit * DV + c]) - decay * hk;   // v - (exp(g) h)^T k
  const float brc = b * rc;
  float acc2 = 0.f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int d = w * kPer + i;
    const float hn = fmaf(ks[d], brc, decay * hc[i]);              // exp(g) h + beta k r^T
    h[(size_t)d * DV] = hn;
    acc2 = fmaf(hn, qs[d], acc2);
  }
  part_q[w][x] = acc2;
  __syncthreads();
  if (w == 0) {
    float ov = 0.f;
#pragma unroll
    for (int y = 0; y < kRows; ++y) ov += part_q[y][x];
    from_f(o + (size_t)unit * DV + c, scale * ov);
  }
}

template <typename T, int DK, int DV>
cudaError_t launch_step(const void* q, const void* k, const void* v, const float* g, const void* beta,
                        float scale, float* state, void* o, int N, int Hqk, int Hv, cudaStream_t st) {
  trace_pre(kKernStep, st);
  constexpr int kCols = cols_for<DK>();
  gdn_step_kernel<T, DK, DV><<<(unsigned)N * (unsigned)Hv * (DV / kCols), dim3(kCols, rows_for<DK>()), 0, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), g, static_cast<const T*>(beta),
      scale, state, static_cast<T*>(o), Hqk, Hv);
  const cudaError_t err = cudaGetLastError();
  trace_post(st);
  return err;
}

template <typename T, int DK>
cudaError_t launch_step_dv(int dv, const void* q, const void* k, const void* v, const float* g, const void* beta,
                           float scale, float* state, void* o, int N, int Hqk, int Hv, cudaStream_t st) {
  if (dv == 256) return launch_step<T, DK, 256>(q, k, v, g, beta, scale, state, o, N, Hqk, Hv, st);
  if (dv == 128) return launch_step<T, DK, 128>(q, k, v, g, beta, scale, state, o, N, Hqk, Hv, st);
  return launch_step<T, DK, 64>(q, k, v, g, beta, scale, state, o, N, Hqk, Hv, st);
}

template <typename T>
cudaError_t launch_step_dims(int dk, int dv, const void* q, const void* k, const void* v, const float* g,
                             const void* beta, float scale, float* state, void* o, int N, int Hqk, int Hv,
                             cudaStream_t st) {
  if (dk == 256) return launch_step_dv<T, 256>(dv, q, k, v, g, beta, scale, state, o, N, Hqk, Hv, st);
  if (dk == 128) return launch_step_dv<T, 128>(dv, q, k, v, g, beta, scale, state, o, N, Hqk, Hv, st);
  return launch_step_dv<T, 64>(dv, q, k, v, g, beta, scale, state, o, N, Hqk, Hv, st);
}

bool head_dim_ok(int d) { return d == 64 || d == 128 || d == 256; }

bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace gdn

extern "C" gdn_status gdn_recurrent_step(gdn_dtype dtype, int N, int Hqk, int Hv, int dk, int dv,
                                         const void* q, const void* k, const void* v, const float* g,
                                         const void* beta, float scale, float* state, void* o,
                                         cudaStream_t stream) {
  if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
  if (N < 0 || Hqk < 1 || Hv < 1 || Hv % Hqk != 0) return GDN_ERR_INVALID_ARG;
  if (!gdn::head_dim_ok(dk) || !gdn::head_dim_ok(dv)) return GDN_ERR_UNSUPPORTED;
  // grid: N Hv dv / (64, or 32 at dk = 256) blocks
  if ((long long)N * Hv * (dv / (dk == 256 ? 32 : 64)) >= (1LL << 31)) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  const void* ptrs[] = {q, k, v, g, beta, state, o};
  for (const void* p : ptrs)
    if (p == nullptr || !gdn::aligned(p)) return GDN_ERR_INVALID_ARG;
  const cudaError_t err =
      dtype == GDN_BF16
          ? gdn::launch_step_dims<__nv_bfloat16>(dk, dv, q, k, v, g, beta, scale, state, o, N, Hqk, Hv, stream)
          : gdn::launch_step_dims<float>(dk, dv, q, k, v, g, beta, scale, state, o, N, Hqk, Hv, stream);
  if (err != cudaSuccess) {
    char msg[160];
    snprintf(msg, sizeof(msg), "recurrent step launch: %s", cudaGetErrorString(err));
    gdn::set_last_error(msg);
    return GDN_ERR_CUDA;
  }
  return GDN_OK;
}
