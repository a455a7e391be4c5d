// Intra-card context parallelism: the segment table of packed sequences and the
// exact affine stitch ("FlashQLA resource", section 3, gate-driven automatic
// intra-card context parallelism: a sequence split into segments that run on
// different SMs).
//
// A segment's end state is an affine function of its start state,
// h_end = M h_start + b, where M (dk x dk) is the segment's transition (its run with
// h_start = I and v = 0) and b its run from a zero state. Chaining these maps over the
// segments of a sequence gives every segment its exact start state.
#include "gdn_common.cuh"
#include "gdn_tc.cuh"

namespace gdn {

constexpr int kPlanThreads = 1024;

// One CTA: per sequence n, its segment count max(1, ceil(chunks_n / seg_chunks)); an
// exclusive scan gives the first pair index of each sequence; the table lists
// (n, seg) for every pair. Inconsistent cu_seqlens are reported in the status word.
__global__ void __launch_bounds__(kPlanThreads)
gdn_cp_plan_kernel(const FwdParams p, int seg_chunks, int max_pairs, int2* table, int* count, int* first_pair,
                   int* chunk_off) {
  __shared__ int part[kPlanThreads];
  const int tid = threadIdx.x;
  const int per = (p.N + kPlanThreads - 1) / kPlanThreads;
  const int n0 = min(p.N, tid * per), n1 = min(p.N, n0 + per);
  int mine = 0;
  for (int n = n0; n < n1; ++n) {
    int lo = p.cu[n], hi = p.cu[n + 1];
    if (lo < 0 || hi < lo || hi > p.T) {
      report_error(p, kDevBadSeqlens);
      hi = lo = 0;
    }
    const int ch = (hi - lo + kChunk - 1) / kChunk;
    mine += max(1, (ch + seg_chunks - 1) / seg_chunks);
  }
  // chunk offsets (exclusive scan of ceil(len / 64)), when asked
  if (chunk_off) {
    int chunks = 0;
    for (int n = n0; n < n1; ++n) {
      int lo = p.cu[n], hi = p.cu[n + 1];
      if (lo < 0 || hi < lo || hi > p.T) hi = lo = 0;
      chunks += (hi - lo + kChunk - 1) / kChunk;
    }
    part[tid] = chunks;
    __syncthreads();
    for (int off = 1; off < kPlanThreads; off <<= 1) {
      const int v = tid >= off ? part[tid - off] : 0;
      __syncthreads();
      part[tid] += v;
      __syncthreads();
    }
    int base = part[tid] - chunks;
    for (int n = n0; n < n1; ++n) {
      chunk_off[n] = base;
      int lo = p.cu[n], hi = p.cu[n + 1];
      if (lo < 0 || hi < lo || hi > p.T) hi = lo = 0;
      base += (hi - lo + kChunk - 1) / kChunk;
    }
    if (tid == kPlanThreads - 1) chunk_off[p.N] = part[tid];
    __syncthreads();
  }
  part[tid] = mine;
  __syncthreads();
  for (int off = 1; off < kPlanThreads; off <<= 1) {   // inclusive scan (Hillis-Steele)
    const int v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int base = part[tid] - mine;
  for (int n = n0; n < n1; ++n) {
    int lo = p.cu[n], hi = p.cu[n + 1];
    if (lo < 0 || hi < lo || hi > p.T) hi = lo = 0;
    const int ch = (hi - lo + kChunk - 1) / kChunk;
    const int segs = max(1, (ch + seg_chunks - 1) / seg_chunks);
    if (first_pair) first_pair[n] = base;
    if (table)
      for (int sgi = 0; sgi < segs; ++sgi)
        if (base + sgi < max_pairs) table[base + sgi] = make_int2(n, sgi);
    base += segs;
  }
  if (tid == kPlanThreads - 1) {
    const int total = part[tid];
    if (count) *count = min(total, max_pairs);
    if ((table && total > max_pairs) || p.cu[0] != 0 || p.cu[p.N] != p.T) report_error(p, kDevBadSeqlens);
  }
}

// Phase 2 of the exact stitch, for one (sequence, v-head) and 8 of the dv columns of the
// state h (columns evolve independently): for s = 2 .. nseg - 1,
//   slot[s] <- M_{s-1} slot[s-1] + slot[s]
// where slot[s] holds b_{s-1} from phase 1 (slot[1] already holds the exact start of
// segment 1, phase 1 having run segment 0 from h0) and M is stored row-major [dk][dk].
// reverse (the backward's state gradient dh = dS^T, carried from the sequence end): slot[s] is the
// gradient at the end of segment s; for s = nseg - 3 .. 0,
//   slot[s] <- M_{s+1} slot[s+1] + slot[s]
// where slot[s] holds c_{s+1} (segment s + 1 run from a zero end gradient) and slot[nseg - 2]
// already holds the exact value (the last segment ran from dhT).
constexpr int kStitchCols = 8;
constexpr int kStitchThreads = 256;

__global__ void __launch_bounds__(kStitchThreads)
gdn_cp_stitch_kernel(const FwdParams p, const TcPlan plan, const int* first_pair, int reverse) {
  __shared__ float hcur[128 * kStitchCols];
  const int groups = 128 / kStitchCols;
  const int cg = blockIdx.x % groups;
  const int unit = blockIdx.x / groups;
  const int j = unit % p.Hv, n = unit / p.Hv;
  int b, s, e;
  if (!seq_span(p, n, b, s, e)) return;
  const int nchunks = (e - s + kChunk - 1) / kChunk;
  const int nseg = max(1, (nchunks + plan.seg_chunks - 1) / plan.seg_chunks);
  if (nseg < 3) return;                              // nothing to chain
  const int pi0 = first_pair ? first_pair[n] : n * plan.max_segs;
  const size_t hsz = 128 * 128;
  const int tid = threadIdx.x;
  const int row = tid >> 1, c4 = (tid & 1) * 4;      // 4 outputs: h[row][c0 + c4 .. +3]
  const int c0 = cg * kStitchCols;
  // forward: the known slot is 1 and the chain runs s = 2 .. nseg - 1 with M_{s-1};
  // reverse: the known slot is nseg - 2 and the chain runs s = nseg - 3 .. 0 with M_{s+1}
  float* slot1 = plan.seg_state + ((size_t)(pi0 + (reverse ? nseg - 2 : 1)) * p.Hv + j) * hsz;
  for (int idx = tid; idx < 128 * kStitchCols; idx += kStitchThreads)
    hcur[idx] = slot1[(size_t)(idx / kStitchCols) * 128 + c0 + idx % kStitchCols];
  __syncthreads();
  for (int step = 0; step < nseg - 2; ++step) {
    const int sg = reverse ? nseg - 3 - step : 2 + step;
    const float* M = plan.seg_trans + ((size_t)(pi0 + (reverse ? sg + 1 : sg - 1)) * p.Hv + j) * hsz;
    float* dst = plan.seg_state + ((size_t)(pi0 + sg) * p.Hv + j) * hsz;
    float acc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] = dst[(size_t)row * 128 + c0 + c4 + u];
    const float4* mrow = reinterpret_cast<const float4*>(M + (size_t)row * 128);
    for (int m4 = 0; m4 < 32; ++m4) {
      const float4 mv = mrow[m4];
      const float mm[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float* hr = hcur + (m4 * 4 + t) * kStitchCols + c4;
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u] = fmaf(mm[t], hr[u], acc[u]);
      }
    }
    __syncthreads();                                  // every thread done reading hcur
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      dst[(size_t)row * 128 + c0 + c4 + u] = acc[u];
      hcur[row * kStitchCols + c4 + u] = acc[u];
    }
    __syncthreads();
  }
}

cudaError_t launch_cp_plan(const FwdParams& p, int seg_chunks, int max_pairs, int2* table, int* count,
                           int* first_pair, int* chunk_off, cudaStream_t st) {
  trace_pre(kKernCpPlan, st);
  gdn_cp_plan_kernel<<<1, kPlanThreads, 0, st>>>(p, seg_chunks, max_pairs, table, count, first_pair, chunk_off);
  cudaError_t err = cudaGetLastError();
  trace_post(st);
  return err;
}

cudaError_t launch_cp_stitch(const FwdParams& p, const TcPlan& plan, const int* first_pair, cudaStream_t st,
                             bool reverse) {
  const int grid = p.N * p.Hv * (128 / kStitchCols);
  trace_pre(kKernCpStitch, st);
  gdn_cp_stitch_kernel<<<grid, kStitchThreads, 0, st>>>(p, plan, first_pair, reverse ? 1 : 0);
  cudaError_t err = cudaGetLastError();
  trace_post(st);
  return err;
}

}  // namespace gdn
