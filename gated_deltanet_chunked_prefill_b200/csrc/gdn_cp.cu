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

// Phase 2 of the exact stitch, for one (sequence, v-head) and 32 of the dv columns of the
// state h (columns evolve independently): for s = 2 .. nseg - 1,
//   slot[s] <- M_{s-1} slot[s-1] + slot[s]
// where slot[s] holds b_{s-1} from phase 1 (slot[1] already holds the exact start of
// segment 1, phase 1 having run segment 0 from h0) and M is stored row-major [dk][dk].
// reverse (the backward's state gradient dh = dS^T, carried from the sequence end): slot[s] is the
// gradient at the end of segment s; for s = nseg - 3 .. 0,
//   slot[s] <- M_{s+1} slot[s+1] + slot[s]
// where slot[s] holds c_{s+1} (segment s + 1 run from a zero end gradient) and slot[nseg - 2]
// already holds the exact value (the last segment ran from dhT).
constexpr int kStitchCols = 32;               // columns of h per CTA
constexpr int kStitchThreads = 256;           // two threads per row of h, kStitchCols / 2 columns each
constexpr int kStitchPer = kStitchCols / 2;

__global__ void __launch_bounds__(kStitchThreads)
gdn_cp_stitch_kernel(const FwdParams p, const TcPlan plan, const int* first_pair, int reverse) {
  __shared__ __align__(16) float hcur[128 * kStitchCols];
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
  const int row = tid >> 1, c4 = (tid & 1) * kStitchPer;   // outputs h[row][c0 + c4 .. + kStitchPer - 1]
  const int c0 = cg * kStitchCols;
  // Slots in chain order: forward s = 1 .. nseg - 1 (start state of segment s, from M_{s-1}),
  // reverse s = nseg - 2 .. 0 (end gradient of segment s, from M_{s+1}). A slot is "direct" when
  // phase 1 already wrote its exact value: forward slot 1 (segment 0 ran from h0), reverse slot
  // nseg - 2 (the last segment ran from dhT), and, with seg_ws, the slot after a segment whose
  // window closes (phase 1 ran that segment from its window). With seg_ws, a segment whose own
  // window closes needs no slot (phase 3 warms it up).
  const int* flags = plan.seg_ws;
  auto closable = [&](int sg) { return flags != nullptr && flags[(size_t)(pi0 + sg) * p.Hv + j] >= 0; };
  for (int step = 0; step < nseg - 1; ++step) {
    const int sg = reverse ? nseg - 2 - step : 1 + step;
    if (closable(sg)) continue;
    const bool direct = reverse ? (sg == nseg - 2 || closable(sg + 1)) : (sg == 1 || closable(sg - 1));
    if (direct) {
      const float* src = plan.seg_state + ((size_t)(pi0 + sg) * p.Hv + j) * hsz;
      __syncthreads();                                // earlier readers of hcur are done
      for (int idx = tid; idx < 128 * kStitchCols; idx += kStitchThreads)
        hcur[idx] = src[(size_t)(idx / kStitchCols) * 128 + c0 + idx % kStitchCols];
      __syncthreads();
      continue;
    }
    const float* M = plan.seg_trans + ((size_t)(pi0 + (reverse ? sg + 1 : sg - 1)) * p.Hv + j) * hsz;
    float* dst = plan.seg_state + ((size_t)(pi0 + sg) * p.Hv + j) * hsz;
    float acc[kStitchPer];
#pragma unroll
    for (int u = 0; u < kStitchPer; ++u) acc[u] = dst[(size_t)row * 128 + c0 + c4 + u];
    const float4* mrow = reinterpret_cast<const float4*>(M + (size_t)row * 128);
    for (int m4 = 0; m4 < 32; ++m4) {
      const float4 mv = mrow[m4];
      const float mm[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float4* hr = reinterpret_cast<const float4*>(hcur + (m4 * 4 + t) * kStitchCols + c4);
#pragma unroll
        for (int u4 = 0; u4 < kStitchPer / 4; ++u4) {
          const float4 h4 = hr[u4];
          acc[4 * u4] = fmaf(mm[t], h4.x, acc[4 * u4]);
          acc[4 * u4 + 1] = fmaf(mm[t], h4.y, acc[4 * u4 + 1]);
          acc[4 * u4 + 2] = fmaf(mm[t], h4.z, acc[4 * u4 + 2]);
          acc[4 * u4 + 3] = fmaf(mm[t], h4.w, acc[4 * u4 + 3]);
        }
      }
    }
    __syncthreads();                                  // every thread done reading hcur
#pragma unroll
    for (int u = 0; u < kStitchPer; ++u) {
      dst[(size_t)row * 128 + c0 + c4 + u] = acc[u];
      hcur[row * kStitchCols + c4 + u] = acc[u];
    }
    __syncthreads();
  }
}

// Gate-driven start with the exact fallback: the window of every segment, once, before phase 1.
// One warp per (pair, v-head). Forward (reverse = 0): the first token of the shortest window of
// whole chunks before the segment's start whose transition bound is <= 2^-64 (at most kMaxWarm
// chunks), else -1; reverse: the end of the window after the segment's end. Each token's factor is
// log(exp(g) max(1, |1 - beta |k|^2|)) (|k|^2 of the normalised row under the q/k normalisation);
// a warp sums a chunk's 64 factors (lanes take tokens l, l + 32) in a fixed order.
constexpr int kProbeWarps = 4;

__device__ __forceinline__ float probe_chunk_bound(const FwdParams& p, int b, int hq, int j, int cs, int n) {
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(p.k);
  const __nv_bfloat16* beta = static_cast<const __nv_bfloat16*>(p.beta);
  const int lane = threadIdx.x & 31;
  float lt = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int tok = lane + 32 * h;
    if (tok < n) {
      const size_t row = (size_t)(b * p.T + cs + tok);
      const uint4* kr = reinterpret_cast<const uint4*>(kg + (row * p.Hqk + hq) * 128);
      float sq = 0.f;
      for (int u = 0; u < 16; ++u) {
        const uint4 v = kr[u];
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const float2 f = __bfloat1622float2(h2[e2]);
          sq = fmaf(f.x, f.x, fmaf(f.y, f.y, sq));
        }
      }
      if (p.qk_l2norm) sq = sq / (sq + 1e-6f);
      const size_t gi = row * p.Hv + j;
      lt += p.g[gi] + __logf(fmaxf(1.f, fabsf(1.f - __bfloat162float(beta[gi]) * sq)));
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) lt += __shfl_xor_sync(0xffffffffu, lt, off);
  return lt;
}

__global__ void __launch_bounds__(32 * kProbeWarps)
gdn_cp_probe_kernel(const FwdParams p, const TcPlan plan, int reverse, int num_items) {
  const int item = blockIdx.x * kProbeWarps + (threadIdx.x >> 5);
  if (item >= num_items) return;
  // every slot is written (-2: no such segment, or no window to look for), so that phase 1 can
  // read a successor's slot before decoding its own item
  WorkItem it;
  if (!get_work_item(p, plan, item, it) || (!reverse && it.seg == 0) ||
      (reverse && it.seg + 1 >= it.segs_used)) {         // plan: kPlanCpP3, one role: item = pi * Hv + j
    if ((threadIdx.x & 31) == 0) plan.seg_ws[item] = -2;
    return;
  }
  const size_t slot = (size_t)it.pi * p.Hv + it.j;
  int w = -1;
  float logb = 0.f;
  if (!reverse) {
    for (int m = 1; m <= kMaxWarm; ++m) {
      const int cs = it.s - m * kChunk;
      if (cs < it.seq_s) break;
      logb += probe_chunk_bound(p, it.b, it.hq, it.j, cs, kChunk);
      if (logb <= kLogWarmBound) { w = cs; break; }
    }
  } else {
    for (int m = 0; m < kMaxWarm; ++m) {
      const int cs = it.e + m * kChunk;
      if (cs >= it.seq_e) break;
      const int n = min(kChunk, it.seq_e - cs);
      logb += probe_chunk_bound(p, it.b, it.hq, it.j, cs, n);
      if (logb <= kLogWarmBound) { w = cs + n; break; }
    }
  }
  if ((threadIdx.x & 31) == 0) plan.seg_ws[slot] = w;
}

cudaError_t launch_cp_probe(const FwdParams& p, const TcPlan& plan, int num_items, cudaStream_t st, bool reverse) {
  if (num_items <= 0) return cudaSuccess;
  TcPlan q = plan;
  q.kind = kPlanCpP3;
  q.roles = 1;
  trace_pre(kKernCpProbe, st);
  gdn_cp_probe_kernel<<<(num_items + kProbeWarps - 1) / kProbeWarps, 32 * kProbeWarps, 0, st>>>(p, q, reverse ? 1 : 0,
                                                                                             num_items);
  cudaError_t err = cudaGetLastError();
  trace_post(st);
  return err;
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
