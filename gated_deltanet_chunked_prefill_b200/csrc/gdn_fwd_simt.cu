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
//
// The chunk runs in four barrier-separated phases. The products give each thread a
// register tile (rows ti + 16r, columns tj + 16s) fed by 16-byte shared-memory loads,
// so a load feeds several FMAs instead of one. The substitution runs on one warp, one
// lane per column, with the column's 16-row block in registers: the rows below the
// block's diagonal are applied with independent accumulators, and only the 16 x 16
// diagonal solve is a dependent chain.
#include "gdn_common.cuh"

namespace gdn {

constexpr int kSimtThreads = 256;
constexpr int kSimtSlice = 32;          // dv columns per CTA
constexpr int kSimtLS = kChunk + 4;     // row stride of L and P (16-byte rows)

template <int DK>
struct SimtSmem {
  // Row stride of K and Q: 16-byte rows, and 8 consecutive rows start 4 banks apart, so
  // the 16-byte loads of 8 lanes on consecutive rows cover the 32 banks once.
  static constexpr int kKS = DK + 4;
  static constexpr int kFloats = 2 * kChunk * kKS /*K, Q*/ + 3 * kChunk * kSimtSlice /*V, D, QH*/ +
                                 DK * kSimtSlice /*h*/ + 2 * kChunk * kSimtLS /*L, P*/ +
                                 4 * kChunk /*gam, beta, exp(gam), exp(gam_n - gam)*/;
  static constexpr size_t kBytes = sizeof(float) * kFloats;
};

__device__ __forceinline__ float4 simt_ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void simt_st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

// Four consecutive elements of an input row as fp32 (16-byte aligned for fp32, 8 for bf16).
__device__ __forceinline__ float4 simt_in4(const float* p) { return simt_ld4(p); }
__device__ __forceinline__ float4 simt_in4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 lo, hi;
  memcpy(&lo, &u.x, 4);
  memcpy(&hi, &u.y, 4);
  const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float simt_dot4(float4 a, float4 b, float acc) {
  acc = fmaf(a.x, b.x, acc);
  acc = fmaf(a.y, b.y, acc);
  acc = fmaf(a.z, b.z, acc);
  return fmaf(a.w, b.w, acc);
}

template <typename IO, int DK>
__global__ void __launch_bounds__(kSimtThreads)
gdn_fwd_simt_kernel(FwdParams p) {
  constexpr int S = kSimtSlice;
  constexpr int KS = SimtSmem<DK>::kKS;
  constexpr int LS = kSimtLS;
  const int slice = blockIdx.x, j = blockIdx.y, n = blockIdx.z;
  const int DV = p.dv;
  const int c0 = slice * S;
  const int hq = j / (p.Hv / p.Hqk);
  const int tid = threadIdx.x;
  // register-tile coordinates: rows ti + 16 r, columns tj + 16 s (a warp spans two rows ti)
  const int ti = tid >> 4, tj = tid & 15;

  int b, s, e;
  if (!seq_span(p, n, b, s, e)) return;

  extern __shared__ float4 sm4[];
  float* sm = reinterpret_cast<float*>(sm4);
  float* Ks = sm;                                  // [64][KS]
  float* Qs = Ks + kChunk * KS;                    // [64][KS]
  float* Vs = Qs + kChunk * KS;                    // [64][S]
  float* Ds = Vs + kChunk * S;                     // [64][S]  diag(beta) Y, then D
  float* QH = Ds + kChunk * S;                     // [64][S]  diag(exp(gam)) Q h
  float* Hs = QH + kChunk * S;                     // [DK][S]  state slice, h layout
  float* Ls = Hs + DK * S;                         // [64][LS]
  float* Ps = Ls + kChunk * LS;                    // [64][LS]
  float* gam = Ps + kChunk * LS;                   // [64]
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
    // ---- load the chunk (rows >= nv are zero); warp 0 also forms the gate scalars
    for (int idx = tid; idx < kChunk * DK / 4; idx += kSimtThreads) {
      const int t = idx / (DK / 4), d = (idx % (DK / 4)) * 4;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), qv = kv;
      if (t < nv) {
        const size_t base = ((size_t)(b * p.T + cs + t) * p.Hqk + hq) * DK + d;
        kv = simt_in4(k + base);
        qv = simt_in4(q + base);
      }
      simt_st4(Ks + t * KS + d, kv);
      simt_st4(Qs + t * KS + d, qv);
    }
    for (int idx = tid; idx < kChunk * S / 4; idx += kSimtThreads) {
      const int t = idx / (S / 4), c = (idx % (S / 4)) * 4;
      float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < nv) vv = simt_in4(v + ((size_t)(b * p.T + cs + t) * p.Hv + j) * DV + c0 + c);
      simt_st4(Vs + t * S + c, vv);
    }
    if (tid < 32) {  // tokens 2 lane and 2 lane + 1: inclusive cumsum of g by a warp scan
      float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
      const size_t gi = (size_t)(b * p.T + cs + 2 * tid) * p.Hv + j;
      if (2 * tid < nv) { a0 = p.g[gi]; b0 = to_f32(beta[gi]); }
      if (2 * tid + 1 < nv) { a1 = p.g[gi + p.Hv]; b1 = to_f32(beta[gi + p.Hv]); }
      const float pair = a0 + a1;
      float run = pair;
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, run, off);
        if (tid >= off) run += y;
      }
      const float excl = run - pair;
      const float g0 = excl + a0, g1 = excl + a0 + a1;
      const int last = nv - 1;
      const float gn = __shfl_sync(0xffffffffu, (last & 1) ? g1 : g0, last >> 1);
      gam[2 * tid] = g0;
      gam[2 * tid + 1] = g1;
      bet[2 * tid] = b0;
      bet[2 * tid + 1] = b1;
      eg[2 * tid] = expf(g0);
      eg[2 * tid + 1] = expf(g1);
      egd[2 * tid] = expf(gn - g0);                // the state update's per-token factor
      egd[2 * tid + 1] = expf(gn - g1);
    }
    __syncthreads();
    // ---- L (strictly lower) and P (lower incl. diagonal). Pairs (r, s) with r < s lie
    //      above the diagonal for every (ti, tj) and are not accumulated.
    {
      float kk[10], qk[10];
#pragma unroll
      for (int x = 0; x < 10; ++x) kk[x] = qk[x] = 0.f;
#pragma unroll 2
      for (int d = 0; d < DK; d += 4) {
        float4 kj[4], ki[4], qi[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          kj[r] = simt_ld4(Ks + (tj + 16 * r) * KS + d);
          ki[r] = simt_ld4(Ks + (ti + 16 * r) * KS + d);
          qi[r] = simt_ld4(Qs + (ti + 16 * r) * KS + d);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int c = 0; c <= r; ++c) {
            kk[r * (r + 1) / 2 + c] = simt_dot4(ki[r], kj[c], kk[r * (r + 1) / 2 + c]);
            qk[r * (r + 1) / 2 + c] = simt_dot4(qi[r], kj[c], qk[r * (r + 1) / 2 + c]);
          }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int i = ti + 16 * r, jj = tj + 16 * c;
          float lv = 0.f, pv = 0.f;
          if (c <= r && jj <= i) {
            const float ed = expf(gam[i] - gam[jj]);
            pv = qk[r * (r + 1) / 2 + c] * ed;
            if (jj < i) lv = bet[i] * kk[r * (r + 1) / 2 + c] * ed;
          }
          Ls[i * LS + jj] = lv;
          Ps[i * LS + jj] = pv;
        }
    }
    // ---- diag(beta) Y = diag(beta) (V - diag(exp(gam)) K h) and diag(exp(gam)) Q h
    {
      float ay[4][2], aq[4][2];
#pragma unroll
      for (int r = 0; r < 4; ++r) ay[r][0] = ay[r][1] = aq[r][0] = aq[r][1] = 0.f;
#pragma unroll 2
      for (int d = 0; d < DK; d += 4) {
        float hv[4][2];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          hv[x][0] = Hs[(d + x) * S + tj];
          hv[x][1] = Hs[(d + x) * S + tj + 16];
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 kr = simt_ld4(Ks + (ti + 16 * r) * KS + d);
          const float4 qr = simt_ld4(Qs + (ti + 16 * r) * KS + d);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            ay[r][u] = simt_dot4(kr, make_float4(hv[0][u], hv[1][u], hv[2][u], hv[3][u]), ay[r][u]);
            aq[r][u] = simt_dot4(qr, make_float4(hv[0][u], hv[1][u], hv[2][u], hv[3][u]), aq[r][u]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = ti + 16 * r, c = tj + 16 * u;
          Ds[i * S + c] = bet[i] * (Vs[i * S + c] - eg[i] * ay[r][u]);
          QH[i * S + c] = eg[i] * aq[r][u];
        }
    }
    __syncthreads();
    // ---- forward substitution (I + L) D = diag(beta) Y on warp 0, lane = column, by 16-row
    //      blocks (rows >= nv stay zero: their L rows and right-hand sides are zero)
    if (tid < 32) {
      const int c = tid;
      const int nblk = (nv + 15) >> 4;
      for (int blk = 0; blk < nblk; ++blk) {
        const int r0 = 16 * blk;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = Ds[(r0 + r) * S + c];
        for (int jj = 0; jj < r0; jj += 4) {
          float dj[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) dj[t] = Ds[(jj + t) * S + c];
#pragma unroll
          for (int r = 0; r < 16; ++r) {
            const float4 l = simt_ld4(Ls + (r0 + r) * LS + jj);
            x[r] = fmaf(-l.x, dj[0], x[r]);
            x[r] = fmaf(-l.y, dj[1], x[r]);
            x[r] = fmaf(-l.z, dj[2], x[r]);
            x[r] = fmaf(-l.w, dj[3], x[r]);
          }
        }
#pragma unroll
        for (int r = 1; r < 16; ++r)
#pragma unroll
          for (int t = 0; t < r; ++t) x[r] = fmaf(-Ls[(r0 + r) * LS + r0 + t], x[t], x[r]);
#pragma unroll
        for (int r = 0; r < 16; ++r) Ds[(r0 + r) * S + c] = x[r];
      }
    }
    __syncthreads();
    // ---- O = scale [diag(exp(gam)) Q h + P D] for rows < nv. P is zero above the diagonal,
    //      so the warp's products stop after its last row (ti | 1) + 48 and after row nv - 1.
    {
      float ao[4][2];
#pragma unroll
      for (int r = 0; r < 4; ++r) ao[r][0] = ao[r][1] = 0.f;
      const int jend = min(((ti | 1) + 52) & ~3, (nv + 3) & ~3);
      for (int jj = 0; jj < jend; jj += 4) {
        float dv[4][2];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          dv[t][0] = Ds[(jj + t) * S + tj];
          dv[t][1] = Ds[(jj + t) * S + tj + 16];
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 pr = simt_ld4(Ps + (ti + 16 * r) * LS + jj);
#pragma unroll
          for (int u = 0; u < 2; ++u)
            ao[r][u] = simt_dot4(pr, make_float4(dv[0][u], dv[1][u], dv[2][u], dv[3][u]), ao[r][u]);
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = ti + 16 * r;
        if (i < nv) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int c = tj + 16 * u;
            o[((size_t)(b * p.T + cs + i) * p.Hv + j) * DV + c0 + c] = from_f32<IO>(p.scale * (QH[i * S + c] + ao[r][u]));
          }
        }
      }
    }
    // ---- h' = exp(gam_n) h + (diag(exp(gam_n - gam)) K)^T D; this thread's rows are
    //      4 ti + 64 g + {0..3}, its columns tj and tj + 16
    {
      constexpr int G = DK / 64;
      float ah[G][4][2];
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int x = 0; x < 4; ++x) ah[g][x][0] = ah[g][x][1] = 0.f;
      for (int t = 0; t < nv; ++t) {
        const float w = egd[t];
        const float d0 = w * Ds[t * S + tj], d1 = w * Ds[t * S + tj + 16];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float4 kv = simt_ld4(Ks + t * KS + 4 * ti + 64 * g);
          ah[g][0][0] = fmaf(kv.x, d0, ah[g][0][0]);
          ah[g][0][1] = fmaf(kv.x, d1, ah[g][0][1]);
          ah[g][1][0] = fmaf(kv.y, d0, ah[g][1][0]);
          ah[g][1][1] = fmaf(kv.y, d1, ah[g][1][1]);
          ah[g][2][0] = fmaf(kv.z, d0, ah[g][2][0]);
          ah[g][2][1] = fmaf(kv.z, d1, ah[g][2][1]);
          ah[g][3][0] = fmaf(kv.w, d0, ah[g][3][0]);
          ah[g][3][1] = fmaf(kv.w, d1, ah[g][3][1]);
        }
      }
      const float egn = expf(gam[nv - 1]);
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int idx = (4 * ti + 64 * g + x) * S + tj + 16 * u;
            Hs[idx] = egn * Hs[idx] + ah[g][x][u];
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
