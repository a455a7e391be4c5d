// fp32 CUDA-core forward of the GDN chunked prefill.
//
// Serves fp32 I/O (whose 1e-4 parity bar plain TF32 tensor-core operands cannot
// meet) and head dims of 64. One CTA owns one (sequence, v-head, 32-column slice
// of dv): the columns of the state h = S^T (dk x dv) evolve independently, so a
// slice carries its own part of the recurrence; the dv-independent chunk
// matrices (Gram, decay mask) are recomputed per slice.
//
// Per 64-token chunk (n valid tokens, rows >= n padded with beta = g = 0 so that
// they contribute exactly nothing), with gam the chunk-local inclusive cumsum of g:
//   L  = strict_lower(diag(beta) K K^T * E),  E_ij = exp(gam_i - gam_j)
//   Y  = V - diag(exp(gam)) K h
//   D  solves (I + L) D = diag(beta) Y            (forward substitution)
//   O  = scale [ diag(exp(gam)) Q h + (Q K^T * E * lower_incl) D ]
//   h' = exp(gam_n) h + (diag(exp(gam_n - gam)) K)^T D
// which is the chunk-parallel form of the gated delta rule (WY/UT transform;
// "FlashQLA resource", section 3, "hardware-friendly algebraic reformulation").
#include "gdn_common.cuh"

namespace gdn {

constexpr int kSimtThreads = 256;
constexpr int kSimtSlice = 32;   // dv columns per CTA

template <int DK>
struct SimtSmem {
  static constexpr int kKs = kChunk * (DK + 1);
  static constexpr int kFloats = 2 * kKs + kChunk * kSimtSlice /*V*/ + DK * kSimtSlice /*h*/ +
                                 2 * kChunk * (kChunk + 1) /*L,P*/ + kChunk * kSimtSlice /*D*/ +
                                 4 * kChunk /*gam, beta, exp(gam), exp(gam_n - gam)*/;
  static constexpr size_t kBytes = sizeof(float) * kFloats;
};

template <typename IO, int DK>
__global__ void __launch_bounds__(kSimtThreads)
gdn_fwd_simt_kernel(FwdParams p) {
  constexpr int S = kSimtSlice;
  const int slice = blockIdx.x, j = blockIdx.y, n = blockIdx.z;
  const int DV = p.dv;
  const int c0 = slice * S;
  const int hq = j / (p.Hv / p.Hqk);
  const int tid = threadIdx.x;

  int b, s, e;
  if (!seq_span(p, n, b, s, e)) return;

  extern __shared__ float sm[];
  float* Ks = sm;                                  // [64][DK+1]
  float* Qs = Ks + SimtSmem<DK>::kKs;              // [64][DK+1]
  float* Vs = Qs + SimtSmem<DK>::kKs;              // [64][S]
  float* Hs = Vs + kChunk * S;                     // [DK][S]  state slice, h layout
  float* Ls = Hs + DK * S;                         // [64][65]
  float* Ps = Ls + kChunk * (kChunk + 1);          // [64][65]
  float* Ds = Ps + kChunk * (kChunk + 1);          // [64][S]  Y, then D
  float* gam = Ds + kChunk * S;                    // [64]
  float* bet = gam + kChunk;                       // [64]
  float* eg = bet + kChunk;                        // [64] exp(gam)
  float* egd = eg + kChunk;                        // [64] exp(gam_n - gam)

  const IO* q = static_cast<const IO*>(p.q);
  const IO* k = static_cast<const IO*>(p.k);
  const IO* v = static_cast<const IO*>(p.v);
  const IO* beta = static_cast<const IO*>(p.beta);
  IO* o = static_cast<IO*>(p.o);

  // initial state slice
  for (int idx = tid; idx < DK * S; idx += kSimtThreads) {
    const int d = idx / S, c = idx % S;
    Hs[idx] = p.h0 ? p.h0[((size_t)(n * p.Hv + j) * DK + d) * DV + c0 + c] : 0.f;
  }

  for (int cs = s; cs < e; cs += kChunk) {
    const int nv = min(kChunk, e - cs);
    __syncthreads();
    // ---- load chunk (rows >= nv are zero)
    for (int idx = tid; idx < kChunk * DK; idx += kSimtThreads) {
      const int t = idx / DK, d = idx % DK;
      float kv = 0.f, qv = 0.f;
      if (t < nv) {
        const size_t base = ((size_t)(b * p.T + cs + t) * p.Hqk + hq) * DK + d;
        kv = to_f32(k[base]);
        qv = to_f32(q[base]);
      }
      Ks[t * (DK + 1) + d] = kv;
      Qs[t * (DK + 1) + d] = qv;
    }
    for (int idx = tid; idx < kChunk * S; idx += kSimtThreads) {
      const int t = idx / S, c = idx % S;
      Vs[idx] = t < nv ? to_f32(v[((size_t)(b * p.T + cs + t) * p.Hv + j) * DV + c0 + c]) : 0.f;
    }
    if (tid < kChunk) {
      const bool ok = tid < nv;
      const size_t gi = (size_t)(b * p.T + cs + tid) * p.Hv + j;
      gam[tid] = ok ? p.g[gi] : 0.f;
      bet[tid] = ok ? to_f32(beta[gi]) : 0.f;
    }
    __syncthreads();
    if (tid < 32) {  // inclusive cumsum of g over 64 values: two per lane, warp scan
      float a0 = gam[2 * tid], a1 = gam[2 * tid + 1];
      float pair = a0 + a1, run = pair;
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, run, off);
        if (tid >= off) run += y;
      }
      const float excl = run - pair;
      gam[2 * tid] = excl + a0;
      gam[2 * tid + 1] = excl + a0 + a1;
    }
    __syncthreads();
    if (tid < kChunk) {
      eg[tid] = expf(gam[tid]);
      egd[tid] = expf(gam[nv - 1] - gam[tid]);     // the state update's per-token factor
    }
    // ---- L (strictly lower) and P (lower incl. diagonal)
    for (int idx = tid; idx < kChunk * kChunk; idx += kSimtThreads) {
      const int i = idx / kChunk, jj = idx % kChunk;
      float lv = 0.f, pv = 0.f;
      if (jj <= i) {
        float kk = 0.f, qk = 0.f;
        for (int d = 0; d < DK; ++d) {
          const float kj = Ks[jj * (DK + 1) + d];
          kk += Ks[i * (DK + 1) + d] * kj;
          qk += Qs[i * (DK + 1) + d] * kj;
        }
        const float ed = expf(gam[i] - gam[jj]);
        pv = qk * ed;
        if (jj < i) lv = bet[i] * kk * ed;
      }
      Ls[i * (kChunk + 1) + jj] = lv;
      Ps[i * (kChunk + 1) + jj] = pv;
    }
    // ---- Y = V - diag(exp(gam)) K h
    for (int idx = tid; idx < kChunk * S; idx += kSimtThreads) {
      const int i = idx / S, c = idx % S;
      float acc = 0.f;
      for (int d = 0; d < DK; ++d) acc += Ks[i * (DK + 1) + d] * Hs[d * S + c];
      Ds[idx] = bet[i] * (Vs[idx] - eg[i] * acc);       // diag(beta) Y
    }
    __syncthreads();
    // ---- forward substitution (I + L) D = diag(beta) Y, row by row; 8 partial sums per column.
    //      A column's 8 lanes sit in one warp and rows only read earlier rows of their own column,
    //      so the warps run their columns independently (warp-level ordering per row)
    {
      const int c = tid >> 3, part = tid & 7;
      for (int i = 1; i < kChunk; ++i) {
        float acc = 0.f;
        for (int jj = part; jj < i; jj += 8) acc += Ls[i * (kChunk + 1) + jj] * Ds[jj * S + c];
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        if (part == 0) Ds[i * S + c] -= acc;
        __syncwarp();
      }
    }
    __syncthreads();
    // ---- O = scale [diag(exp(gam)) Q h + P D]
    for (int idx = tid; idx < kChunk * S; idx += kSimtThreads) {
      const int i = idx / S, c = idx % S;
      if (i >= nv) continue;
      float qh = 0.f, pd = 0.f;
      for (int d = 0; d < DK; ++d) qh += Qs[i * (DK + 1) + d] * Hs[d * S + c];
      for (int jj = 0; jj <= i; ++jj) pd += Ps[i * (kChunk + 1) + jj] * Ds[jj * S + c];
      o[((size_t)(b * p.T + cs + i) * p.Hv + j) * DV + c0 + c] =
          from_f32<IO>(p.scale * (eg[i] * qh + pd));
    }
    __syncthreads();
    // ---- h' = exp(gam_n) h + (diag(exp(gam_n - gam)) K)^T D
    {
      const float egn = expf(gam[nv - 1]);
      for (int idx = tid; idx < DK * S; idx += kSimtThreads) {
        const int d = idx / S, c = idx % S;
        float acc = 0.f;
        for (int t = 0; t < nv; ++t) acc += egd[t] * Ks[t * (DK + 1) + d] * Ds[t * S + c];
        Hs[idx] = egn * Hs[idx] + acc;
      }
    }
  }
  __syncthreads();
  if (p.hT) {
    for (int idx = tid; idx < DK * S; idx += kSimtThreads) {
      const int d = idx / S, c = idx % S;
      p.hT[((size_t)(n * p.Hv + j) * DK + d) * DV + c0 + c] = Hs[idx];
    }
  }
}

template <typename IO, int DK>
static cudaError_t launch_simt_t(const FwdParams& p, cudaStream_t st) {
  auto kern = gdn_fwd_simt_kernel<IO, DK>;
  const size_t smem = SimtSmem<DK>::kBytes;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid(p.dv / kSimtSlice, p.Hv, p.N);
  trace_pre(kKernFwdSimt, st);
  kern<<<grid, kSimtThreads, smem, st>>>(p);
  err = cudaGetLastError();
  trace_post(st);
  return err;
}

cudaError_t launch_fwd_simt(const FwdParams& p, bool bf16, cudaStream_t st) {
  if (bf16) return p.dk == 64 ? launch_simt_t<__nv_bfloat16, 64>(p, st) : launch_simt_t<__nv_bfloat16, 128>(p, st);
  return p.dk == 64 ? launch_simt_t<float, 64>(p, st) : launch_simt_t<float, 128>(p, st);
}

}  // namespace gdn
