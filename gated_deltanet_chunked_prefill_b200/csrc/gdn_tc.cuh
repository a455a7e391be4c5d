// Work decomposition of the tensor-core forward: which token range of which
// (sequence, v-head) a CTA runs, where its initial state comes from and where its
// final state goes.
#pragma once

#include <cuda.h>

#include "gdn_common.cuh"

namespace gdn {

// TMA map of a [rows, heads, 128] bf16 tensor: boxes of box_rows rows x 64 elements of one
// head, 128-byte swizzle (rows = B * T tokens; boxes past the last row read zeros).
bool make_tile_map(CUtensorMap* m, const void* base, int heads, long long rows, int box_rows = 64);

// Outputs and scratch of the backward's gradient kernel.
struct BwdOut {
  void* dq;                  // [B,T,Hqk,dk] bf16
  void* dk;                  // [B,T,Hqk,dk] bf16
  void* dv;                  // [B,T,Hv,dv] bf16
  float* dg;                 // [B,T,Hv]
  void* dbeta;               // [B,T,Hv] bf16
  const void* dO;            // [B,T,Hv,dv] bf16
  const __nv_bfloat16* dstates;   // per-chunk dS' (bf16, dv x dk)
  const float* chunk_a;           // per-chunk A = (I + L)^-1 (fp32, 64 x 64), from the forward pass
  const uint8_t* chunk_p;         // per-chunk P (bf16 swizzled 8 KB tile), from the forward pass
  int qk_partial;            // grouped values: dq/dk go through fp32 per-v-head partials
  float* dq_part;            // [B,T,Hv,dk] fp32
  float* dk_part;            // [B,T,Hv,dk] fp32
};
cudaError_t launch_bwd_grad(const FwdParams& p, const BwdOut& out, long long total_chunks, cudaStream_t st,
                            const char** what);

enum InitMode : int { kInitZero = 0, kInitPtr = 1, kInitIdentity = 2 };

// Grid decomposition chosen on the host (see gdn_api.cu).
//   kPlanUnits:  one CTA per (sequence, v-head); items = N * Hv.
//   kPlanCpP1:   context parallelism, phase 1: per (sequence, v-head, segment s < nseg-1)
//                two CTAs: role 0 runs segment s from a zero state (segment 0: from h0)
//                and stores its end state b_s; role 1 (s >= 1 only) runs it from the
//                identity with v = 0 and stores the segment's transition M_s.
//   kPlanCpP3:   phase 3: per (sequence, v-head, segment) one CTA runs the segment from
//                its stitched start state and writes o (and hT for the last segment).
//   kPlanGate:   gate-driven context parallelism in one launch: per (sequence, v-head,
//                segment) one CTA writes o for its segment; it reconstructs its start state
//                by running, from a zero state, a window of earlier chunks whose decay bound
//                is below 2^-64 (or from the sequence start when no such window exists
//                within kMaxWarm chunks).
enum PlanKind : int { kPlanUnits = 0, kPlanCpP1 = 1, kPlanCpP3 = 2, kPlanGate = 3 };

constexpr int kMaxWarm = 16;                      // longest warm-up window, in chunks
constexpr float kLogWarmBound = -44.3614195558f;  // ln(2^-64)

// A segment is named by its pair index pi: pi = n * max_segs + seg for B independent
// sequences, or the position of (n, seg) in a table the plan kernel builds for packed
// sequences (ordered by n, then seg, so that segment seg + 1 of n is pi + 1).
struct TcPlan {
  int kind;
  int seg_chunks;        // chunks per segment (CP)
  int max_segs;          // segment slots per sequence (B independent sequences)
  int roles;             // 2 in phase 1 of the exact stitch, else 1
  const int2* table;     // nullable: (sequence, segment) per pair index (packed sequences)
  const int* table_count;
  float* seg_state;      // [pairs][Hv][dk][dv] fp32: start state of segment pi (exact stitch)
  float* seg_trans;      // [pairs][Hv][dk][dk] fp32: transition of segment pi (exact stitch)
  // Gate-driven start with the exact stitch as its fallback (nullable; phases 1 and 3 and the
  // stitch): [pairs][Hv] the first token of segment pi's warm-up window when its window closes,
  // else -1 (the segment then starts from its stitched state). Reverse chain: the window's end.
  int* seg_ws;
};

struct WorkItem {
  int n, j, hq, b, s, e;  // sequence, v-head, q/k head, batch row, token range [s, e)
  int seq_s, seq_e;       // token range of the whole sequence
  int seg, segs_used, pi, role;   // context-parallel plans: segment, segments of the sequence, pair, role
  bool gate;              // may start earlier than s with a warm-up window (kPlanGate)
  int init_mode;
  const float* init;      // [dk][dv] fp32 when init_mode == kInitPtr
  float* fin;             // [dk][dv] fp32 destination of the end state, or nullptr
  bool write_o;
  bool zero_v;            // run with v = 0 (transition role)
};

// reverse: the item of the backward's reverse chain under the exact stitch (kPlanCpP1 / kPlanCpP3),
// where the state gradient runs from a segment's end to its start. There p.h0 is dhT and p.hT is
// dh0 (the chain's parameter mapping), `init` is the gradient at the segment end and `fin` receives
// the gradient at its start:
//   kPlanCpP1, segment seg >= 1: role 0 runs from a zero end gradient (the last segment: from dhT)
//     and stores its start gradient in the end slot of segment seg - 1 (pair pi - 1); role 1
//     (seg <= nseg - 2) runs from the identity with dO = 0 and stores the segment's transition.
//   kPlanCpP3: every segment runs from its stitched end gradient (the last: dhT), segment 0 writes
//     dh0.
__device__ __forceinline__ bool get_work_item(const FwdParams& p, const TcPlan& plan, int item, WorkItem& w,
                                              bool reverse = false) {
  const size_t hsz = (size_t)p.dk * p.dv;
  w.write_o = false;
  w.zero_v = false;
  w.fin = nullptr;
  w.init = nullptr;
  w.init_mode = kInitZero;
  w.gate = false;
  w.seg = 0;
  w.segs_used = 1;
  w.pi = 0;
  w.role = 0;
  if (plan.kind == kPlanUnits) {
    w.j = item % p.Hv;
    w.n = item / p.Hv;
    if (!seq_span(p, w.n, w.b, w.s, w.e)) return false;
    w.seq_s = w.s;
    w.seq_e = w.e;
    w.hq = w.j / (p.Hv / p.Hqk);
    if (p.h0) { w.init_mode = kInitPtr; w.init = p.h0 + ((size_t)w.n * p.Hv + w.j) * hsz; }
    if (p.hT) w.fin = p.hT + ((size_t)w.n * p.Hv + w.j) * hsz;
    w.write_o = true;
    return true;
  }
  // context-parallel plans: item = (pi * roles + role) * Hv + j (consecutive items are the
  // v-heads of one segment, so heads that share q/k read the same tiles close in time)
  w.j = item % p.Hv;
  const int rest = item / p.Hv;
  const int role = rest % plan.roles;
  const int pi = rest / plan.roles;
  int seg;
  if (plan.table) {
    if (pi >= *plan.table_count) return false;
    const int2 e = plan.table[pi];
    w.n = e.x;
    seg = e.y;
  } else {
    w.n = pi / plan.max_segs;
    seg = pi % plan.max_segs;
    if (w.n >= p.N) return false;
  }
  int b, s, e;
  if (!seq_span(p, w.n, b, s, e)) return false;
  const int nchunks = (e - s + kChunk - 1) / kChunk;
  const int nseg = (nchunks + plan.seg_chunks - 1) / plan.seg_chunks;
  const int segs_used = nseg > 0 ? nseg : 1;
  if (seg >= segs_used) return false;
  w.b = b;
  w.seq_s = s;
  w.seq_e = e;
  w.hq = w.j / (p.Hv / p.Hqk);
  w.s = s + seg * plan.seg_chunks * kChunk;
  w.e = min(e, w.s + plan.seg_chunks * kChunk);
  w.seg = seg;
  w.segs_used = segs_used;
  w.pi = pi;
  w.role = role;
  const float* h0u = p.h0 ? p.h0 + ((size_t)w.n * p.Hv + w.j) * hsz : nullptr;
  if (reverse) {
    const bool last = seg + 1 == segs_used;
    if (plan.kind == kPlanCpP1) {
      if (seg == 0) return false;                           // its start gradient comes from phase 3
      if (role == 0) {
        if (last && h0u) { w.init_mode = kInitPtr; w.init = h0u; }
        w.fin = plan.seg_state + ((size_t)(pi - 1) * p.Hv + w.j) * hsz;
      } else {
        if (last) return false;                             // the last segment ends at dhT
        w.init_mode = kInitIdentity;
        w.zero_v = true;
        w.fin = plan.seg_trans + ((size_t)pi * p.Hv + w.j) * (size_t)p.dk * p.dk;
      }
      return true;
    }
    if (role != 0) return false;
    if (!last) { w.init_mode = kInitPtr; w.init = plan.seg_state + ((size_t)pi * p.Hv + w.j) * hsz; }
    else if (h0u) { w.init_mode = kInitPtr; w.init = h0u; }
    if (seg == 0 && p.hT) w.fin = p.hT + ((size_t)w.n * p.Hv + w.j) * hsz;
    w.write_o = true;
    return true;
  }
  if (plan.kind == kPlanCpP1) {
    if (seg + 1 >= segs_used) return false;                 // last segment: no map needed
    if (role == 0) {
      if (seg == 0 && h0u) { w.init_mode = kInitPtr; w.init = h0u; }
      w.fin = plan.seg_state + ((size_t)(pi + 1) * p.Hv + w.j) * hsz;   // b_seg -> slot of seg + 1
    } else {
      if (seg == 0) return false;                           // segment 0 starts from the known h0
      w.init_mode = kInitIdentity;
      w.zero_v = true;
      w.fin = plan.seg_trans + ((size_t)pi * p.Hv + w.j) * (size_t)p.dk * p.dk;
    }
    return true;
  }
  // phase 3 of the exact stitch, or the single launch of the gate-driven plan
  if (role != 0) return false;
  w.gate = plan.kind == kPlanGate;
  if (seg == 0) {
    if (h0u) { w.init_mode = kInitPtr; w.init = h0u; }
  } else if (plan.kind == kPlanCpP3) {
    w.init_mode = kInitPtr;
    w.init = plan.seg_state + ((size_t)pi * p.Hv + w.j) * hsz;
  }
  if (seg + 1 == segs_used && p.hT) w.fin = p.hT + ((size_t)w.n * p.Hv + w.j) * hsz;
  w.write_o = true;
  return true;
}

// Sum over the tokens [cs, cs + n) (n <= 64) of log(exp(g_t) max(1, |1 - beta_t |k_t|^2|)),
// the log of the exact spectral norm of each token's state transition exp(g)(I - beta k k^T)
// (eigenvalues exp(g) and exp(g)(1 - beta |k|^2)). Under the q/k normalisation k is the
// normalised row, |k|^2 = s / (s + eps) for the raw squared norm s. All 512 threads of the CTA
// call it and get the same value; wsum is 16 floats of shared scratch.
__device__ __forceinline__ float chunk_log_bound(const FwdParams& p, const WorkItem& it, int cs, int n,
                                                 float* wsum) {
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(p.k);
  const __nv_bfloat16* beta = static_cast<const __nv_bfloat16*>(p.beta);
  const int tok = threadIdx.x >> 3, part = threadIdx.x & 7;   // 64 tokens x 8 threads
  float sq = 0.f;
  const size_t row = (size_t)(it.b * p.T + cs + tok);
  if (tok < n) {
    const uint4* kr = reinterpret_cast<const uint4*>(kg + (row * p.Hqk + it.hq) * 128 + part * 16);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint4 v = kr[u];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        sq = fmaf(f.x, f.x, fmaf(f.y, f.y, sq));
      }
    }
  }
  sq += __shfl_xor_sync(0xffffffffu, sq, 1);
  sq += __shfl_xor_sync(0xffffffffu, sq, 2);
  sq += __shfl_xor_sync(0xffffffffu, sq, 4);
  if (p.qk_l2norm) sq = sq / (sq + 1e-6f);
  float lt = 0.f;
  if (part == 0 && tok < n) {
    const size_t gi = row * p.Hv + it.j;
    const float bt = __bfloat162float(beta[gi]);
    lt = p.g[gi] + __logf(fmaxf(1.f, fabsf(1.f - bt * sq)));
  }
  lt += __shfl_xor_sync(0xffffffffu, lt, 8);
  lt += __shfl_xor_sync(0xffffffffu, lt, 16);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = lt;   // warp w covers tokens 4w .. 4w + 3
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int u = 0; u < 16; ++u) tot += wsum[u];
  __syncthreads();
  return tot;
}

// First token of the shortest window of whole chunks before token `s` (at most kMaxWarm, within the
// sequence) whose transition has spectral norm <= 2^-64, or -1 if there is none. CTA-wide.
__device__ __forceinline__ int gate_window_start(const FwdParams& p, const WorkItem& it, int s, float* wsum) {
  float logb = 0.f;
  for (int m = 1; m <= kMaxWarm; ++m) {
    const int cs = s - m * kChunk;
    if (cs < it.seq_s) break;
    logb += chunk_log_bound(p, it, cs, kChunk, wsum);
    if (logb <= kLogWarmBound) return cs;
  }
  return -1;
}

// Reverse chain: the end (exclusive) of the shortest window of chunks after token `e` (at most
// kMaxWarm, within the sequence) whose transition bound is <= 2^-64 (the adjoint's norm equals
// the transition's), or -1. CTA-wide.
__device__ __forceinline__ int gate_window_end(const FwdParams& p, const WorkItem& it, int e, float* wsum) {
  float logb = 0.f;
  for (int m = 0; m < kMaxWarm; ++m) {
    const int cs = e + m * kChunk;
    if (cs >= it.seq_e) break;
    const int n = min(kChunk, it.seq_e - cs);
    logb += chunk_log_bound(p, it, cs, n, wsum);
    if (logb <= kLogWarmBound) return cs + n;
  }
  return -1;
}

cudaError_t launch_fwd_tc(const FwdParams& p, const TcPlan& plan, int num_items, cudaStream_t st,
                          const char** what);
// Backward, reverse state-gradient chain (see gdn_bwd_chain.cu for the parameter mapping).
cudaError_t launch_bwd_chain(const FwdParams& p, const TcPlan& plan, int num_items, cudaStream_t st,
                             const char** what);
// Packed sequences: build the (sequence, segment) table of a segmented plan.
cudaError_t launch_cp_plan(const FwdParams& p, int seg_chunks, int max_pairs, int2* table, int* count,
                           int* first_pair, int* chunk_off, cudaStream_t st);
// Exact stitch, phase 2: chain the segment maps h_{s+1} = M_s h_s + b_s in place; reverse (the
// backward's state gradient): dh_end(s) = M_{s+1} dh_end(s + 1) + c_{s+1}, from the sequence end.
// Gate-driven start with the exact fallback: the window of every segment and v-head into plan.seg_ws
// (forward: before the segment's start; reverse: after its end), before phase 1.
cudaError_t launch_cp_probe(const FwdParams& p, const TcPlan& plan, int num_items, cudaStream_t st, bool reverse);
// With plan.seg_ws (gate-driven start with the exact fallback) only the segments whose window does
// not close are chained; a segment whose predecessor's end state came straight from phase 1 (the
// sequence start, or a window that closes) restarts the chain.
cudaError_t launch_cp_stitch(const FwdParams& p, const TcPlan& plan, const int* first_pair, cudaStream_t st,
                             bool reverse = false);

}  // namespace gdn
