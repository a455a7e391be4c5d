// Work decomposition of the tensor-core forward: which token range of which
// (sequence, v-head) a CTA runs, where its initial state comes from and where its
// final state goes.
#pragma once

#include "gdn_common.cuh"

namespace gdn {

enum InitMode : int { kInitZero = 0, kInitPtr = 1, kInitIdentity = 2 };

// Grid decomposition chosen on the host (see gdn_api.cu).
//   kPlanUnits:  one CTA per (sequence, v-head); items = N * Hv.
//   kPlanCpP1:   context parallelism, phase 1: per (sequence, v-head, segment s < nseg-1)
//                two CTAs: role 0 runs segment s from a zero state (segment 0: from h0)
//                and stores its end state b_s; role 1 (s >= 1 only) runs it from the
//                identity with v = 0 and stores the segment's transition M_s.
//   kPlanCpP3:   phase 3: per (sequence, v-head, segment) one CTA runs the segment from
//                its stitched start state and writes o (and hT for the last segment).
enum PlanKind : int { kPlanUnits = 0, kPlanCpP1 = 1, kPlanCpP3 = 2 };

struct TcPlan {
  int kind;
  int seg_chunks;        // chunks per segment (CP)
  int max_segs;          // segment slots per sequence in the workspace
  float* seg_state;      // [N][Hv][max_segs][dk][dv] fp32: start state of segment s (s >= 1)
  float* seg_trans;      // [N][Hv][max_segs][dk][dk] fp32: transition M_s of segment s (s >= 1)
};

struct WorkItem {
  int n, j, hq, b, s, e;  // sequence, v-head, q/k head, batch row, token range [s, e)
  int init_mode;
  const float* init;      // [dk][dv] fp32 when init_mode == kInitPtr
  float* fin;             // [dk][dv] fp32 destination of the end state, or nullptr
  bool write_o;
  bool zero_v;            // run with v = 0 (transition role)
};

__device__ __forceinline__ bool get_work_item(const FwdParams& p, const TcPlan& plan, int item, WorkItem& w) {
  const size_t hsz = (size_t)p.dk * p.dv;
  w.write_o = false;
  w.zero_v = false;
  w.fin = nullptr;
  w.init = nullptr;
  w.init_mode = kInitZero;
  if (plan.kind == kPlanUnits) {
    w.j = item % p.Hv;
    w.n = item / p.Hv;
    if (!seq_span(p, w.n, w.b, w.s, w.e)) return false;
    w.hq = w.j / (p.Hv / p.Hqk);
    if (p.h0) { w.init_mode = kInitPtr; w.init = p.h0 + ((size_t)w.n * p.Hv + w.j) * hsz; }
    if (p.hT) w.fin = p.hT + ((size_t)w.n * p.Hv + w.j) * hsz;
    w.write_o = true;
    return true;
  }
  // context-parallel plans: item = ((n * Hv + j) * max_segs + seg) * roles + role
  const int roles = plan.kind == kPlanCpP1 ? 2 : 1;
  const int role = item % roles;
  int rest = item / roles;
  const int seg = rest % plan.max_segs;
  rest /= plan.max_segs;
  w.j = rest % p.Hv;
  w.n = rest / p.Hv;
  int b, s, e;
  if (!seq_span(p, w.n, b, s, e)) return false;
  const int nchunks = (e - s + kChunk - 1) / kChunk;
  const int nseg = (nchunks + plan.seg_chunks - 1) / plan.seg_chunks;
  const int segs_used = nseg > 0 ? nseg : 1;
  if (seg >= segs_used) return false;
  w.b = b;
  w.hq = w.j / (p.Hv / p.Hqk);
  w.s = s + seg * plan.seg_chunks * kChunk;
  w.e = min(e, w.s + plan.seg_chunks * kChunk);
  if (w.s > e) w.s = e;
  const size_t slot = ((size_t)w.n * p.Hv + w.j) * plan.max_segs;
  if (plan.kind == kPlanCpP1) {
    if (seg + 1 >= segs_used) return false;                 // last segment: no transition needed
    if (role == 0) {
      if (seg == 0 && p.h0) { w.init_mode = kInitPtr; w.init = p.h0 + ((size_t)w.n * p.Hv + w.j) * hsz; }
      w.fin = plan.seg_state + (slot + seg + 1) * hsz;      // b_s lands in the next segment's slot
    } else {
      if (seg == 0) return false;                           // segment 0 starts from the known h0
      w.init_mode = kInitIdentity;
      w.zero_v = true;
      w.fin = plan.seg_trans + (slot + seg) * (size_t)p.dk * p.dk;
    }
    return true;
  }
  // phase 3
  if (seg == 0) {
    if (p.h0) { w.init_mode = kInitPtr; w.init = p.h0 + ((size_t)w.n * p.Hv + w.j) * hsz; }
  } else {
    w.init_mode = kInitPtr;
    w.init = plan.seg_state + (slot + seg) * hsz;
  }
  if (seg + 1 == segs_used && p.hT) w.fin = p.hT + ((size_t)w.n * p.Hv + w.j) * hsz;
  w.write_o = true;
  return true;
}

cudaError_t launch_fwd_tc(const FwdParams& p, const TcPlan& plan, int num_items, cudaStream_t st,
                          const char** what);

}  // namespace gdn
