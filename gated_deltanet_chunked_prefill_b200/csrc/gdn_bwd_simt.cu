// CUDA-core backward of the GDN chunked prefill for the sizes the tensor-core kernels do not
// take (fp32 I/O, head dims of 64): the exact token-level adjoint of the recurrence, per
// (sequence, v-head), with the forward states recomputed from checkpoints.
//
//   forward, per token:  h~ = exp(g) h;  r = v - h~^T k;  h = h~ + beta k r^T   (h = S^T, dk x dv)
//   adjoint, in reverse token order, with dh the adjoint of the state after the token:
//     dh += scale q do^T;   dq = scale h do = scale (h~ do + beta k (r . do))
//     dbeta = k^T dh r;     dr = beta dh^T k;   dv = dr
//     dk = beta dh r - h~ dr;   dh~ = dh - k dr^T;   dg = <dh~, h~>;   dh <- exp(g) dh~
// dh starts at dhT (or 0) and ends as dh0. This is the recurrence the pages' chunked kernels
// evaluate ("Qwen's FlashQLA targets the expensive bit of long-context AI", "What happened";
// "FlashQLA resource", section 3), differentiated token by token.
//
// A persistent CTA takes (sequence, v-head) units in turn. Phase 1 runs the sequence forward and
// stores the state at every 64th token (fp32, one slot per 64-token block of every sequence, the
// slot order of the chunk-state cache). Phase 2 walks the blocks backward: it recomputes the
// block's h~ and r token by token into the CTA's own buffer, then runs the adjoint over them.
// Shared memory holds h (or h~) and dh as [dk][dv + 1] (padded). In the column passes four lanes
// of a warp share each state column, each walking a quarter of its rows, and in the row passes
// four lanes share each row; two xor shuffles combine the quarters. The block buffer keeps h~ in
// thread order, so its writes are coalesced and each token's h~ is loaded into registers one
// token ahead of its adjoint. Every reduction runs in a fixed order (bit-reproducible).
#include <algorithm>

#include "gdn_common.cuh"

namespace gdn {

namespace {

constexpr int kBwdSimtThreads = 256;
constexpr int kBlk = 64;               // tokens between checkpoints

struct BwdSimtArgs {
  const void* dO;        // [B,T,Hv,dv] (IO)
  const float* dhT;      // nullable [N,Hv,dk,dv]
  void* dq;              // [B,T,Hqk,dk] (IO), written directly when Hv == Hqk
  void* dk;
  float* dq_part;        // [B,T,Hv,dk] fp32 per v-head when Hv > Hqk (summed afterwards), else null
  float* dk_part;
  void* dv;              // [B,T,Hv,dv] (IO)
  float* dg;             // [B,T,Hv]
  void* dbeta;           // [B,T,Hv] (IO)
  float* dh0;            // nullable [N,Hv,dk,dv]
  float* ckpt;           // [slots][Hv][dk][dv]: the state before every 64th token of each sequence
  float* tok;            // per CTA: [64][dk][dv] h~ of the block's tokens, then [64][dv] their r
};

template <int DK, int DV>
struct BwdSimtSmem {
  static constexpr int kLd = DV + 1;
  static constexpr int kFloats = 2 * DK * kLd + 2 * DK /*k, q*/ + 4 * DV /*v|do, r, dr, spare*/ +
                                 2 * kBwdSimtThreads /*reductions*/ + 8;
  static constexpr size_t kBytes = sizeof(float) * kFloats;
};

// sum of red[0 .. kBwdSimtThreads) in a fixed order (warp shuffles, then the warps' partials);
// every thread returns the total. Called by all threads.
__device__ __forceinline__ float block_sum(float x, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  if (lane == 0) red[warp] = x;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kBwdSimtThreads / 32; ++w) t += red[w];
  __syncthreads();
  return t;
}

__device__ __forceinline__ int block_sum_int(int x, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  int* ired = reinterpret_cast<int*>(red);
  if (lane == 0) ired[warp] = x;
  __syncthreads();
  int t = 0;
#pragma unroll
  for (int w = 0; w < kBwdSimtThreads / 32; ++w) t += ired[w];
  __syncthreads();
  return t;
}

// Sum over the four lanes qg = lane >> 3 that share lane & 7 (two xor steps). Floating-point
// addition is commutative, so all four lanes hold the same bits afterwards.
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 8);
  x += __shfl_xor_sync(0xffffffffu, x, 16);
  return x;
}

template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(kBwdSimtThreads)
gdn_bwd_simt_kernel(const FwdParams p, const BwdSimtArgs a) {
  constexpr int LD = BwdSimtSmem<DK, DV>::kLd;
  constexpr int NC = DV / 64;          // column sets of a thread in the column passes
  constexpr int NR = DK / 64;          // row sets of a thread in the row passes
  constexpr int NE = (DK / 4) * NC;    // state elements a thread owns in the column passes
  extern __shared__ float sm[];
  float* H = sm;                       // [DK][LD]  h, or h~ of the token being differentiated
  float* DH = H + DK * LD;             // [DK][LD]  dh
  float* ks = DH + DK * LD;            // [DK]
  float* qs = ks + DK;                 // [DK]
  float* vs = qs + DK;                 // [DV]  v (recompute) or do (adjoint)
  float* rs = vs + DV;                 // [DV]  r
  float* drs = rs + DV;                // [DV]  dr
  float* red = drs + 2 * DV;           // reductions
  float* scal = red + 2 * kBwdSimtThreads;   // g, beta of the token

  const int tid = threadIdx.x;
  // State-pass coordinates. Column passes: this thread's columns are cb + 64 cs (cs < NC) and
  // its rows 4 i + qg (i < DK / 4); row passes swap the roles (rows cb + 64 s, s < NR; columns
  // 4 i + qg). The four lanes qg of one column (row) are lanes (lane & 7) + 8 qg of one warp, and
  // at every step the 32 lanes of a warp touch 32 distinct banks (LD = 1 mod 32).
  const int lane = tid & 31, warp = tid >> 5;
  const int qg = lane >> 3;
  const int cb = (warp & 3) + 32 * (warp >> 2) + 4 * (lane & 7);
  const IO* q = static_cast<const IO*>(p.q);
  const IO* k = static_cast<const IO*>(p.k);
  const IO* v = static_cast<const IO*>(p.v);
  const IO* dO = static_cast<const IO*>(a.dO);
  const IO* beta = static_cast<const IO*>(p.beta);
  const size_t S = (size_t)DK * DV;
  // this CTA's block buffer: h~ of each token in thread order (element e of thread tid at
  // e * kBwdSimtThreads + tid, e = i * NC + cs for row 4 i + qg and column cb + 64 cs), then r
  float* tokh = a.tok + (size_t)blockIdx.x * (kBlk * S + kBlk * DV);
  float* tokr = tokh + kBlk * S;
  const int units = p.N * p.Hv;
  const int nblk_dense = (p.T + kBlk - 1) / kBlk;

  for (int unit = blockIdx.x; unit < units; unit += gridDim.x) {
    const int n = unit / p.Hv, j = unit % p.Hv;
    const int hq = j / (p.Hv / p.Hqk);
    int b, s, e;
    if (!seq_span(p, n, b, s, e)) continue;          // uniform over the CTA
    const int Tn = e - s;
    // first checkpoint slot of sequence n (the chunk-state cache's slot order)
    int slot0 = n * nblk_dense;
    if (p.cu != nullptr) {
      int part = 0;
      for (int m = tid; m < n; m += kBwdSimtThreads) part += (p.cu[m + 1] - p.cu[m] + kBlk - 1) / kBlk;
      slot0 = block_sum_int(part, red);
    }
    auto row_of = [&](int t) { return (size_t)b * p.T + s + t; };
    // A token's inputs travel through registers one token ahead (every thread holds at most one
    // element of k, q and v or do: DK, DV <= kBwdSimtThreads), so that their load latency overlaps
    // the previous token's passes; publish() puts them in shared memory (the caller then syncs).
    struct Tok {
      float k, q, v, g, b;
    };
    static_assert(DK <= kBwdSimtThreads && DV <= kBwdSimtThreads, "one element per thread");
    auto fetch = [&](int t, bool adjoint) {
      Tok x{0.f, 0.f, 0.f, 0.f, 0.f};
      if (t < 0 || t >= Tn) return x;
      const size_t row = row_of(t);
      if (tid < DK) {
        x.k = to_f32(k[(row * p.Hqk + hq) * DK + tid]);
        if (adjoint) x.q = to_f32(q[(row * p.Hqk + hq) * DK + tid]);
      }
      if (tid < DV) x.v = to_f32(adjoint ? dO[(row * p.Hv + j) * DV + tid] : v[(row * p.Hv + j) * DV + tid]);
      if (tid == 0) {
        x.g = p.g[row * p.Hv + j];
        x.b = to_f32(beta[row * p.Hv + j]);
      }
      return x;
    };
    auto publish = [&](const Tok& x, bool adjoint) {
      if (tid < DK) {
        ks[tid] = x.k;
        if (adjoint) qs[tid] = x.q;
      }
      if (tid < DV) vs[tid] = x.v;
      if (tid == 0) {
        scal[0] = x.g;
        scal[1] = x.b;
      }
    };
    // one forward token on H (column pass); with `keep`, h~ and r go to the block buffer at i
    auto forward_token = [&](bool keep, int i) {
      const float eg = __expf(scal[0]), bt = scal[1];
#pragma unroll
      for (int cs = 0; cs < NC; ++cs) {
        const int r = cb + 64 * cs;
        float u0 = 0.f, u1 = 0.f;
#pragma unroll
        for (int x = 0; x < DK / 4; x += 2) {
          u0 = fmaf(H[(4 * x + qg) * LD + r], ks[4 * x + qg], u0);
          u1 = fmaf(H[(4 * x + 4 + qg) * LD + r], ks[4 * x + 4 + qg], u1);
        }
        const float rr = vs[r] - eg * quad_sum(u0 + u1);
        if (keep && qg == 0) tokr[i * DV + r] = rr;
#pragma unroll
        for (int x = 0; x < DK / 4; ++x) {
          const int d = 4 * x + qg;
          const float ht = eg * H[d * LD + r];
          if (keep) tokh[(size_t)i * S + (size_t)(x * NC + cs) * kBwdSimtThreads + tid] = ht;
          H[d * LD + r] = fmaf(bt * ks[d], rr, ht);
        }
      }
    };

    // ---- phase 1: forward over the sequence, the state before every 64th token to its slot
    for (int idx = tid; idx < DK * DV; idx += kBwdSimtThreads) {
      const int d = idx / DV, r = idx % DV;
      H[d * LD + r] = p.h0 ? p.h0[((size_t)unit * DK + d) * DV + r] : 0.f;
    }
    __syncthreads();
    Tok nx = fetch(0, false);
    for (int t = 0; t < Tn; ++t) {
      if (t % kBlk == 0) {
        float* c = a.ckpt + ((size_t)(slot0 + t / kBlk) * p.Hv + j) * S;
        for (int idx = tid; idx < DK * DV; idx += kBwdSimtThreads) c[idx] = H[(idx / DV) * LD + idx % DV];
      }
      publish(nx, false);
      nx = fetch(t + 1, false);
      __syncthreads();
      forward_token(false, 0);
      __syncthreads();
    }

    // ---- phase 2: the adjoint, block by block from the end
    for (int idx = tid; idx < DK * DV; idx += kBwdSimtThreads) {
      const int d = idx / DV, r = idx % DV;
      DH[d * LD + r] = a.dhT ? a.dhT[((size_t)unit * DK + d) * DV + r] : 0.f;
    }
    float hnext[NE];                   // h~ of the next token to differentiate (own elements), and its r
    float rnext = 0.f;
    auto load_tok = [&](int i) {
#pragma unroll
      for (int x = 0; x < NE; ++x) hnext[x] = tokh[(size_t)i * S + (size_t)x * kBwdSimtThreads + tid];
      if (tid < DV) rnext = tokr[i * DV + tid];
    };
    for (int blk = (Tn + kBlk - 1) / kBlk - 1; blk >= 0; --blk) {
      const int t0 = blk * kBlk, nt = min(kBlk, Tn - t0);
      __syncthreads();
      const float* c = a.ckpt + ((size_t)(slot0 + blk) * p.Hv + j) * S;
      for (int idx = tid; idx < DK * DV; idx += kBwdSimtThreads) H[(idx / DV) * LD + idx % DV] = c[idx];
      __syncthreads();
      nx = fetch(t0, false);
      for (int i = 0; i < nt; ++i) {               // recompute h~, r of the block's tokens
        publish(nx, false);
        nx = fetch(i + 1 < nt ? t0 + i + 1 : -1, false);
        __syncthreads();
        forward_token(true, i);
        __syncthreads();
      }
      nx = fetch(t0 + nt - 1, true);
      load_tok(nt - 1);
      for (int i = nt - 1; i >= 0; --i) {
        const int t = t0 + i;
        const size_t row = row_of(t);
        publish(nx, true);
        nx = fetch(i > 0 ? t - 1 : -1, true);
#pragma unroll
        for (int x = 0; x < NE; ++x) H[(4 * (x / NC) + qg) * LD + cb + 64 * (x % NC)] = hnext[x];
        if (tid < DV) rs[tid] = rnext;
        if (i > 0) load_tok(i - 1);                // in flight during this token's passes
        __syncthreads();
        const float eg = __expf(scal[0]), bt = scal[1];
        // columns: dh += scale q do^T;  dr = beta dh^T k
#pragma unroll
        for (int cs = 0; cs < NC; ++cs) {
          const int r = cb + 64 * cs;
          const float dor = p.scale * vs[r];
          float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
          for (int x = 0; x < DK / 4; x += 2) {
            const int d0 = 4 * x + qg, d1 = d0 + 4;
            const float x0 = fmaf(qs[d0], dor, DH[d0 * LD + r]);
            const float x1 = fmaf(qs[d1], dor, DH[d1 * LD + r]);
            DH[d0 * LD + r] = x0;
            DH[d1 * LD + r] = x1;
            acc0 = fmaf(x0, ks[d0], acc0);
            acc1 = fmaf(x1, ks[d1], acc1);
          }
          const float acc = quad_sum(acc0 + acc1);
          if (qg == 0) drs[r] = bt * acc;
        }
        __syncthreads();
        // rows: dq = scale (h~ do + beta k (r . do)), dk = beta dh r - h~ dr, dbeta = k^T dh r
        float bpart = 0.f;
#pragma unroll
        for (int rsx = 0; rsx < NR; ++rsx) {
          const int d = cb + 64 * rsx;
          float w = 0.f, a1 = 0.f, a2 = 0.f, rd = 0.f;
#pragma unroll
          for (int x = 0; x < DV / 4; ++x) {
            const int r = 4 * x + qg;
            const float hh = H[d * LD + r];
            w = fmaf(DH[d * LD + r], rs[r], w);
            a1 = fmaf(hh, vs[r], a1);
            a2 = fmaf(hh, drs[r], a2);
            rd = fmaf(rs[r], vs[r], rd);
          }
          w = quad_sum(w);
          a1 = quad_sum(a1);
          a2 = quad_sum(a2);
          rd = quad_sum(rd);
          if (qg == 0) {
            const float dqv = p.scale * fmaf(bt * ks[d], rd, a1);
            const float dkv = bt * w - a2;
            bpart = fmaf(ks[d], w, bpart);
            if (a.dq_part) {
              a.dq_part[(row * p.Hv + j) * DK + d] = dqv;
              a.dk_part[(row * p.Hv + j) * DK + d] = dkv;
            } else {
              static_cast<IO*>(a.dq)[(row * p.Hqk + hq) * DK + d] = from_f32<IO>(dqv);
              static_cast<IO*>(a.dk)[(row * p.Hqk + hq) * DK + d] = from_f32<IO>(dkv);
            }
          }
        }
        const float dbeta = block_sum(bpart, red);
        // columns: dh~ = dh - k dr^T;  dg = <dh~, h~>;  dh <- exp(g) dh~;  dv = dr
        float gpart = 0.f;
#pragma unroll
        for (int cs = 0; cs < NC; ++cs) {
          const int r = cb + 64 * cs;
          const float drr = drs[r];
          float g0 = 0.f, g1 = 0.f;
#pragma unroll
          for (int x = 0; x < DK / 4; x += 2) {
            const int d0 = 4 * x + qg, d1 = d0 + 4;
            const float x0 = DH[d0 * LD + r] - ks[d0] * drr;
            const float x1 = DH[d1 * LD + r] - ks[d1] * drr;
            g0 = fmaf(x0, H[d0 * LD + r], g0);
            g1 = fmaf(x1, H[d1 * LD + r], g1);
            DH[d0 * LD + r] = eg * x0;
            DH[d1 * LD + r] = eg * x1;
          }
          const float gt = quad_sum(g0 + g1);
          if (qg == 0) {
            gpart += gt;
            static_cast<IO*>(a.dv)[(row * p.Hv + j) * DV + r] = from_f32<IO>(drr);
          }
        }
        const float dg = block_sum(gpart, red);
        if (tid == 0) {
          a.dg[row * p.Hv + j] = dg;
          static_cast<IO*>(a.dbeta)[row * p.Hv + j] = from_f32<IO>(dbeta);
        }
      }
    }
    __syncthreads();
    if (a.dh0) {
      for (int idx = tid; idx < DK * DV; idx += kBwdSimtThreads)
        a.dh0[(size_t)unit * S + idx] = DH[(idx / DV) * LD + idx % DV];
    }
    __syncthreads();
  }
}

// fp32 per-v-head partials of dq / dk -> the sum over the v-heads of each q/k head (fixed order)
template <typename IO>
__global__ void gdn_bwd_simt_reduce_kernel(const float* __restrict__ part, IO* __restrict__ out, long long rows,
                                           int Hv, int Hqk, int dk) {
  const int G = Hv / Hqk;
  const long long total = rows * Hqk * dk;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int d = (int)(idx % dk);
    const long long rh = idx / dk;
    const int hq = (int)(rh % Hqk);
    const long long row = rh / Hqk;
    float acc = 0.f;
    for (int jj = 0; jj < G; ++jj) acc += part[(row * Hv + hq * G + jj) * dk + d];
    out[idx] = from_f32<IO>(acc);
  }
}

template <typename IO, int DK, int DV>
cudaError_t launch_typed(const FwdParams& p, const BwdSimtArgs& a, int grid, cudaStream_t st) {
  constexpr size_t smem = BwdSimtSmem<DK, DV>::kBytes;
  cudaError_t err = cudaFuncSetAttribute(gdn_bwd_simt_kernel<IO, DK, DV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  trace_pre(kKernBwdSimt, st);
  gdn_bwd_simt_kernel<IO, DK, DV><<<grid, kBwdSimtThreads, smem, st>>>(p, a);
  err = cudaGetLastError();
  trace_post(st);
  if (err != cudaSuccess || !a.dq_part) return err;
  const long long rows = (long long)p.B * p.T;
  const long long total = rows * p.Hqk * DK;
  const int blocks = (int)std::min<long long>((total + 255) / 256, 4096);
  trace_pre(kKernBwdReduce, st);
  gdn_bwd_simt_reduce_kernel<IO><<<blocks, 256, 0, st>>>(a.dq_part, static_cast<IO*>(a.dq), rows, p.Hv, p.Hqk, DK);
  gdn_bwd_simt_reduce_kernel<IO><<<blocks, 256, 0, st>>>(a.dk_part, static_cast<IO*>(a.dk), rows, p.Hv, p.Hqk, DK);
  err = cudaGetLastError();
  trace_post(st);
  return err;
}

template <typename IO>
cudaError_t launch_io(const FwdParams& p, const BwdSimtArgs& a, int grid, cudaStream_t st) {
  if (p.dk == 64 && p.dv == 64) return launch_typed<IO, 64, 64>(p, a, grid, st);
  if (p.dk == 64 && p.dv == 128) return launch_typed<IO, 64, 128>(p, a, grid, st);
  if (p.dk == 128 && p.dv == 64) return launch_typed<IO, 128, 64>(p, a, grid, st);
  return launch_typed<IO, 128, 128>(p, a, grid, st);
}

}  // namespace

// Bytes of the per-CTA block buffer of the CUDA-core backward.
size_t bwd_simt_tok_bytes(int dk, int dv) { return sizeof(float) * ((size_t)kBlk * dk * dv + (size_t)kBlk * dv); }

// The CUDA-core backward: `grid` persistent CTAs (each with bwd_simt_tok_bytes of `tok`), then,
// with grouped values, the dq / dk sums over the v-heads.
cudaError_t launch_bwd_simt(const FwdParams& p, bool bf16, const void* dO, const float* dhT, void* dq, void* dk,
                            float* dq_part, float* dk_part, void* dv, float* dg, void* dbeta, float* dh0,
                            float* ckpt, float* tok, int grid, cudaStream_t st) {
  BwdSimtArgs a{dO, dhT, dq, dk, dq_part, dk_part, dv, dg, dbeta, dh0, ckpt, tok};
  return bf16 ? launch_io<__nv_bfloat16>(p, a, grid, st) : launch_io<float>(p, a, grid, st);
}

}  // namespace gdn
