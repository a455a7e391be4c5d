// C-ABI entry points: argument validation, workspace layout, planning, launches.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "gdn_common.cuh"
#include "gdn_tc.cuh"

namespace gdn {
cudaError_t launch_fwd_simt(const FwdParams& p, bool bf16, cudaStream_t st);
size_t bwd_simt_tok_bytes(int dk, int dv);
cudaError_t launch_bwd_simt(const FwdParams& p, bool bf16, const void* dO, const float* dhT, void* dq, void* dk,
                            float* dq_part, float* dk_part, void* dv, float* dg, void* dbeta, float* dh0,
                            float* ckpt, float* tok, int grid, cudaStream_t st);
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


constexpr int kTraceMax = 4096;
struct Trace {
  cudaEvent_t events[2 * kTraceMax];
  int capacity = 0;   // > 0 while a trace is active
  int count = 0;
  int ids[kTraceMax];
};
thread_local Trace g_trace;
thread_local long long g_launches = 0;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

bool uses_tc(gdn_dtype dtype, const Shape& s) { return dtype == GDN_BF16 && s.dk == 128 && s.dv == 128; }

// The caller's options with the defaults (all zero) filled in; GDN_ERR_INVALID_ARG for a value
// outside its range.
gdn_status read_options(const gdn_options* opt, gdn_options& o) {
  o = gdn_options{};
  if (opt) o = *opt;
  for (int r : o.reserved)
    if (r != 0) return GDN_ERR_INVALID_ARG;
  if (o.deterministic != 0 && o.deterministic != 1) return GDN_ERR_INVALID_ARG;
  if (o.qk_l2norm != 0 && o.qk_l2norm != 1) return GDN_ERR_INVALID_ARG;
  if (o.test_stall != 0 && o.test_stall != 1) return GDN_ERR_INVALID_ARG;
  if (o.cp_mode < -1) return GDN_ERR_INVALID_ARG;
  if (o.cp_exact < 0 || o.cp_exact > 2) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

// Segment length (chunks) the options ask for: n > 0 segments of n chunks, -1 off, 0 automatic.
// cp_segment_chunks, when nonzero, wins; cp_mode = n > 0 gives at most n segments per sequence.
int segment_option(const Shape& s, const gdn_options* opt) {
  if (!opt) return 0;
  if (opt->cp_segment_chunks != 0) return opt->cp_segment_chunks < 0 ? -1 : opt->cp_segment_chunks;
  if (opt->cp_mode < 0) return -1;
  if (opt->cp_mode > 0) {
    const int nch = (s.T + kChunk - 1) / kChunk;
    return nch > 0 ? (nch + opt->cp_mode - 1) / opt->cp_mode : -1;
  }
  return 0;
}

// Status of a device status word's code.
gdn_status device_code_status(int code) {
  switch (code) {
    case kDevOk: return GDN_OK;
    case kDevTimeout: return GDN_ERR_DEVICE_TIMEOUT;
    case kDevMisaligned: return GDN_ERR_DEVICE_LAUNCH;
    default: return GDN_ERR_DEVICE_INPUT;
  }
}

// Row coordinates of the per-chunk state arrays (slots x Hv x 128 rows) are 32-bit TMA
// coordinates: refuse sizes whose last row does not fit.
bool state_rows_fit(long long slots, int Hv) { return slots * Hv * 128LL < (1LL << 31); }

// Segment length (chunks) for automatic context parallelism, 0 = none. Independent
// sequences: the segment count minimising waves x (segment chunks + 1 warm-up chunk),
// with one CTA per SM per wave. Packed sequences (lengths unknown on the host): segments
// of 32 chunks once the batch holds at least 128 chunks.
int auto_segment(const Shape& s, int nch) {
  const int sms = num_sms();
  if (s.packed) return nch >= 128 ? 32 : 0;
  const long long units = (long long)s.N * s.Hv;
  long long best_cost = -1;
  int best = 1;
  for (int nseg = 1; nseg <= 64 && nseg <= nch; ++nseg) {
    const long long waves = (units * nseg + sms - 1) / sms;
    const long long cost = waves * ((nch + nseg - 1) / nseg + (nseg > 1 ? 1 : 0));
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = nseg; }
  }
  return best > 1 ? (nch + best - 1) / best : 0;
}

struct FwdPlan {
  int kind = kPlanUnits;
  int seg_chunks = 0, max_segs = 0, max_pairs = 0;
  bool table = false;
  bool exact = false;      // exact affine stitch for every segment
  bool fallback = false;   // gate-driven start, the exact stitch where a segment's window does not close
  size_t off_table = 0, off_count = 0, off_first = 0, off_state = 0, off_trans = 0, off_ws = 0;
  size_t total = kStatusBytes;
  bool phased() const { return exact || fallback; }   // the three-phase launch sequence
  size_t off_chunk_off = 0;     // packed sequences: per-sequence first chunk slot (state cache)
};

FwdPlan plan_forward(gdn_dtype dtype, const Shape& s, const gdn_options* opt) {
  FwdPlan f;
  if (!uses_tc(dtype, s) || s.T == 0) return f;
  if (s.packed) {
    f.off_chunk_off = f.total;
    f.total = align256(f.total + (size_t)(s.N + 1) * sizeof(int));
  }
  const int mode = segment_option(s, opt);
  if (mode < 0) return f;
  const int nch = (s.T + kChunk - 1) / kChunk;
  const int seg = mode > 0 ? mode : auto_segment(s, nch);
  if (seg <= 0 || (!s.packed && seg >= nch)) return f;
  f.seg_chunks = seg;
  // cp_exact: 0 gate-driven start, restarting at the sequence start where a window does not close;
  // 1 exact stitch; 2 gate-driven with the exact stitch as that fallback, once a sequence can have 3
  // or more segments (with 2, the fallback's two phases take as long as the restart).
  const int cpx = opt ? opt->cp_exact : 0;
  f.exact = cpx == 1;
  f.fallback = cpx == 2 && (nch + seg - 1) / seg >= 3;
  f.kind = f.phased() ? kPlanCpP3 : kPlanGate;
  if (s.packed) {
    f.table = true;
    f.max_pairs = (nch + s.N + seg - 1) / seg + s.N;
  } else {
    f.max_segs = (nch + seg - 1) / seg;
    f.max_pairs = s.N * f.max_segs;
  }
  size_t off = f.total;
  if (f.table) {
    f.off_table = off; off = align256(off + (size_t)f.max_pairs * sizeof(int2));
    f.off_count = off; off = align256(off + sizeof(int));
    f.off_first = off; off = align256(off + (size_t)s.N * sizeof(int));
  }
  if (f.phased()) {
    const size_t per = (size_t)f.max_pairs * s.Hv * s.dk * s.dv * sizeof(float);
    f.off_state = off; off = align256(off + per);
    f.off_trans = off; off = align256(off + per);
  }
  if (f.fallback) {
    f.off_ws = off; off = align256(off + (size_t)f.max_pairs * s.Hv * sizeof(int));
  }
  f.total = off;
  return f;
}

// The chunk-state cache (gdn_options.states): the bf16 start states of every chunk slot,
// then the fp32 A = (I + L)^-1 of every chunk slot.
long long state_slots(const Shape& s) {
  const long long nch = (s.T + kChunk - 1) / kChunk;
  return s.packed ? nch + s.N : (long long)s.N * nch;
}
size_t cache_states_bytes(const Shape& s) { return (size_t)state_slots(s) * s.Hv * s.dk * s.dv * 2; }
size_t cache_a_bytes(const Shape& s) { return (size_t)state_slots(s) * s.Hv * kChunk * kChunk * sizeof(float); }
// then the bf16 P = lower_incl(Q K^T * E) tile of every chunk slot (8 KB, swizzled as the operand)
size_t cache_p_bytes(const Shape& s) { return (size_t)state_slots(s) * s.Hv * kChunk * kChunk * 2; }

// The CUDA-core backward (fp32 I/O or head dims 64): fp32 state checkpoints every 64 tokens (the
// cache's slot order), one 64-token block buffer per persistent CTA, and with grouped values the
// per-v-head dq / dk partials.
struct SimtBwdPlan {
  int grid = 1;
  size_t off_ckpt = 0, off_tok = 0, off_dq = 0, off_dk = 0, total = 0;
};
SimtBwdPlan plan_backward_simt(const Shape& s) {
  SimtBwdPlan b;
  const long long units = (long long)s.N * s.Hv;
  b.grid = (int)std::max<long long>(1, std::min<long long>(units, num_sms()));
  size_t off = kStatusBytes;
  b.off_ckpt = off;
  off = align256(off + (size_t)state_slots(s) * s.Hv * s.dk * s.dv * sizeof(float));
  b.off_tok = off;
  off = align256(off + (size_t)b.grid * bwd_simt_tok_bytes(s.dk, s.dv));
  if (s.Hv != s.Hqk) {
    const size_t part = (size_t)s.B * s.T * s.Hv * s.dk * sizeof(float);
    b.off_dq = off;
    off = align256(off + part);
    b.off_dk = off;
    off = align256(off + part);
  }
  b.total = off;
  return b;
}

// Workspace of gdn_chunk_bwd for one reading of the shape: the tensor-core plan (bf16, dk = dv = 128)
// and, without a chunk-state cache, the CUDA-core plan (the size query does not know the dtype).
size_t bwd_workspace_for(const Shape& s, const gdn_options* opt);

struct BwdPlan {
  FwdPlan chain;                 // gate-driven segments (or none) for the two sequential passes
  long long total_chunks = 0;    // chunk slots (upper bound for packed sequences)
  bool grouped = false;
  size_t off_chunk_off = 0, off_states = 0, off_dstates = 0, off_a = 0, off_p = 0, off_dq = 0, off_dk = 0;
  size_t total = kStatusBytes;
};

BwdPlan plan_backward(const Shape& s, const gdn_options* opt) {
  BwdPlan b;
  b.chain = plan_forward(GDN_BF16, s, opt);     // the segments of both sequential passes
  const int nch = (s.T + kChunk - 1) / kChunk;
  b.total_chunks = s.packed ? (long long)nch + s.N : (long long)s.N * nch;
  b.grouped = s.Hv != s.Hqk;
  size_t off = b.chain.total;
  if (s.packed) b.off_chunk_off = b.chain.off_chunk_off;
  const size_t st = (size_t)b.total_chunks * s.Hv * s.dk * s.dv * 2;
  if (!(opt && opt->states)) {                  // states and A are in the caller's cache otherwise
    b.off_states = off; off = align256(off + st);
    b.off_a = off; off = align256(off + (size_t)b.total_chunks * s.Hv * kChunk * kChunk * sizeof(float));
    b.off_p = off; off = align256(off + (size_t)b.total_chunks * s.Hv * kChunk * kChunk * 2);
  }
  b.off_dstates = off; off = align256(off + st);

  if (b.grouped) {
    const size_t part = (size_t)s.B * s.T * s.Hv * s.dk * sizeof(float);
    b.off_dq = off; off = align256(off + part);
    b.off_dk = off; off = align256(off + part);
  }
  b.total = off;
  return b;
}

size_t bwd_workspace_for(const Shape& s, const gdn_options* opt) {
  size_t total = kStatusBytes;
  if (s.dk == 128 && s.dv == 128) total = plan_backward(s, opt).total;
  if (!(opt && opt->states)) total = std::max(total, plan_backward_simt(s).total);
  return total;
}

}  // namespace

namespace {
// ---- host-buffer calls (gdn_chunk_host)

// Scratch layout: device copies of every input and output, then the chunk-state cache (forward +
// backward) and the workspaces, each 256-byte aligned. Offsets in bytes from the scratch base;
// n_* are array sizes in bytes.
struct HostLayout {
  size_t q = 0, k = 0, v = 0, g = 0, beta = 0, h0 = 0, cu = 0, dO = 0, dhT = 0;
  size_t o = 0, hT = 0, dq = 0, dk = 0, dv = 0, dg = 0, dbeta = 0, dh0 = 0;
  size_t states = 0, ws_f = 0, ws_b = 0;
  size_t n_qk = 0, n_v = 0, n_g = 0, n_beta = 0, n_h = 0, n_cu = 0;
  size_t ws_f_bytes = 0, ws_b_bytes = 0, total = 0;
};

HostLayout host_layout(gdn_dtype dtype, const Shape& s, bool fw, bool bw, const gdn_options& op) {
  HostLayout L;
  const size_t es = dtype == GDN_F32 ? 4 : 2;
  const size_t tok = (size_t)s.B * s.T;
  L.n_qk = tok * s.Hqk * s.dk * es;
  L.n_v = tok * s.Hv * s.dv * es;
  L.n_g = tok * s.Hv * sizeof(float);
  L.n_beta = tok * s.Hv * es;
  L.n_h = (size_t)s.N * s.Hv * s.dk * s.dv * sizeof(float);
  L.n_cu = (size_t)(s.N + 1) * sizeof(int32_t);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.q = take(L.n_qk); L.k = take(L.n_qk); L.v = take(L.n_v); L.g = take(L.n_g); L.beta = take(L.n_beta);
  L.h0 = take(L.n_h); L.cu = take(L.n_cu);
  if (bw) { L.dO = take(L.n_v); L.dhT = take(L.n_h); }
  if (fw) { L.o = take(L.n_v); L.hT = take(L.n_h); }
  if (bw) {
    L.dq = take(L.n_qk); L.dk = take(L.n_qk); L.dv = take(L.n_v); L.dg = take(L.n_g); L.dbeta = take(L.n_beta);
    L.dh0 = take(L.n_h);
  }
  gdn_options plan_opt = op;
  plan_opt.states = nullptr;
  if (fw && bw && uses_tc(dtype, s)) {   // the cache exists on the tensor-core path only
    L.states = take(cache_states_bytes(s) + cache_a_bytes(s) + cache_p_bytes(s));
    plan_opt.states = &L;           // the backward plans without its own state pass (only non-null matters)
  }
  if (fw) { L.ws_f_bytes = plan_forward(dtype, s, &plan_opt).total; L.ws_f = take(L.ws_f_bytes); }
  if (bw) {
    L.ws_b_bytes = uses_tc(dtype, s) ? plan_backward(s, &plan_opt).total : plan_backward_simt(s).total;
    L.ws_b = take(L.ws_b_bytes);
  }
  L.total = off;
  return L;
}

// Events that order calls sharing a scratch buffer, created on its first use on a device.
struct HostEvents {
  int device = -1;
  bool used = false;                 // an earlier call recorded compute_done and out_done
  int in_use = 0;                    // calls enqueuing on these events right now (never swept then)
  cudaEvent_t in_fwd = nullptr, in_bwd = nullptr, fwd_done = nullptr, compute_done = nullptr, out_done = nullptr;
};
std::mutex g_host_mu;
std::unordered_map<const void*, HostEvents>& host_event_map() {
  static auto* m = new std::unordered_map<const void*, HostEvents>();   // lives as long as the process
  return *m;
}

// A scratch address whose recorded work has all completed needs no ordering any more: its events
// can go. Swept when the table grows past a few dozen addresses (a caller that allocates a new
// scratch for every call would otherwise grow it without bound).
bool host_events_idle(const HostEvents& e) {
  cudaEvent_t evs[] = {e.in_fwd, e.in_bwd, e.fwd_done, e.compute_done, e.out_done};
  for (cudaEvent_t ev : evs) {
    const cudaError_t q = ev ? cudaEventQuery(ev) : cudaSuccess;
    if (q != cudaSuccess) {
      cudaGetLastError();            // not ready (or never recorded on this device): keep it
      return false;
    }
  }
  return true;
}
void host_events_sweep(const void* keep) {
  auto& m = host_event_map();
  if (m.size() <= 64) return;
  for (auto it = m.begin(); it != m.end();) {
    if (it->first != keep && it->second.in_use == 0 && host_events_idle(it->second)) {
      cudaEvent_t evs[] = {it->second.in_fwd, it->second.in_bwd, it->second.fwd_done, it->second.compute_done,
                           it->second.out_done};
      for (cudaEvent_t ev : evs)
        if (ev) cudaEventDestroy(ev);
      it = m.erase(it);
    } else {
      ++it;
    }
  }
}

gdn_status host_events(const void* scratch, HostEvents*& out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail("gdn_chunk_host: cudaGetDevice", err);
  std::lock_guard<std::mutex> lock(g_host_mu);
  host_events_sweep(scratch);
  HostEvents& e = host_event_map()[scratch];
  if (e.device != dev) {             // first use, or the address now belongs to another device
    cudaEvent_t* evs[] = {&e.in_fwd, &e.in_bwd, &e.fwd_done, &e.compute_done, &e.out_done};
    for (cudaEvent_t* ev : evs) {
      if (*ev) cudaEventDestroy(*ev);
      *ev = nullptr;
    }
    e.device = -1;
    e.used = false;
    for (cudaEvent_t* ev : evs) {
      err = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
      if (err != cudaSuccess) return cuda_fail("gdn_chunk_host: cudaEventCreate", err);
    }
    e.device = dev;
  }
  ++e.in_use;
  out = &e;
  return GDN_OK;
}

// Releases a scratch address's events at the end of the call that took them (host_events).
struct HostEventsHold {
  HostEvents* e = nullptr;
  ~HostEventsHold() {
    if (e) {
      std::lock_guard<std::mutex> lock(g_host_mu);
      --e->in_use;
    }
  }
};
}  // namespace

// The library's per-device status word (gdn_check_device_error): kernels record their first
// finding here as well as in the call's workspace.
__device__ int g_device_status;

namespace {
// Device address of the per-device status word on the current device, or nullptr when it cannot
// be found (the call then records in its workspace only). Looked up on every call: the host-side
// name of a __device__ variable is not a device address, and an address cached across a
// cudaDeviceReset would be stale.
int* device_status_word() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_device_status) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return static_cast<int*>(ptr);
}
}  // namespace

namespace gdn {
void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

void trace_pre(int kernel_id, cudaStream_t st) {
  ++g_launches;
  Trace& t = g_trace;
  if (t.count < t.capacity) {
    t.ids[t.count] = kernel_id;
    cudaEventRecord(t.events[2 * t.count], st);
  }
}
void trace_post(cudaStream_t st) {
  Trace& t = g_trace;
  if (t.count < t.capacity) {
    cudaEventRecord(t.events[2 * t.count + 1], st);
    ++t.count;
  }
}
}  // namespace gdn

extern "C" {

gdn_status gdn_trace_begin(int capacity) {
  Trace& t = g_trace;
  if (t.capacity > 0 || capacity <= 0 || capacity > kTraceMax) return GDN_ERR_INVALID_ARG;
  for (int i = 0; i < 2 * capacity; ++i) {
    cudaError_t err = cudaEventCreate(&t.events[i]);
    if (err != cudaSuccess) {
      for (int k = 0; k < i; ++k) cudaEventDestroy(t.events[k]);
      return cuda_fail("trace event create", err);
    }
  }
  t.capacity = capacity;
  t.count = 0;
  return GDN_OK;
}

int gdn_trace_end(float* ms, int* kernel_ids) {
  Trace& t = g_trace;
  const int n = t.count;
  int ret = n;
  for (int i = 0; i < n; ++i) {
    float v = 0.f;
    if (cudaEventSynchronize(t.events[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&v, t.events[2 * i], t.events[2 * i + 1]) != cudaSuccess)
      ret = -1;
    if (ms) ms[i] = v;
    if (kernel_ids) kernel_ids[i] = t.ids[i];
  }
  for (int i = 0; i < 2 * t.capacity; ++i) cudaEventDestroy(t.events[i]);
  t.capacity = 0;
  t.count = 0;
  return ret;
}

const char* gdn_kernel_name(int kernel_id) {
  static const char* names[kKernCount] = {"gdn_fwd_tc_kernel",   "gdn_fwd_simt_kernel", "gdn_cp_stitch_kernel",
                                          "gdn_bwd_grad_kernel", "gdn_bwd_simt_kernel", "gdn_bwd_reduce_kernel",
                                          "gdn_cp_plan_kernel",  "gdn_bwd_chain_kernel", "gdn_step_kernel",
                                          "gdn_cp_probe_kernel"};
  return (kernel_id >= 0 && kernel_id < kKernCount) ? names[kernel_id] : "unknown";
}

long long gdn_launch_count(void) { return g_launches; }

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
    case GDN_ERR_DEVICE_LAUNCH: return "a kernel found its launch unusable (shared memory misaligned)";
  }
  return "unknown status";
}

size_t gdn_chunk_fwd_workspace_size(int B, int T, int Hqk, int Hv, int dk, int dv, int num_seqs,
                                    const gdn_options* opt) {
  // sized for both the bf16 tensor-core plan (the larger) and the fp32 path. B == 1 with
  // num_seqs >= 1 fits both a packed call and a call without cu_seqlens (whose num_seqs is ignored).
  Shape s;
  size_t total = kStatusBytes;
  if (check_shape(B, T, Hqk, Hv, dk, dv, 0, false, s) == GDN_OK) total = plan_forward(GDN_BF16, s, opt).total;
  if (num_seqs > 0 && B == 1 && check_shape(B, T, Hqk, Hv, dk, dv, num_seqs, true, s) == GDN_OK)
    total = std::max(total, plan_forward(GDN_BF16, s, opt).total);
  return total;
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
  gdn_options op;
  st = read_options(opt, op);
  if (st != GDN_OK) return st;
  opt = &op;
  if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARG;
  void* save_states = op.states;
  if ((save_states || op.qk_l2norm) && !uses_tc(dtype, s)) return GDN_ERR_UNSUPPORTED;
  if (save_states && !state_rows_fit(state_slots(s), s.Hv)) return GDN_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, g, beta, h0, cu_seqlens, o, hT, save_states};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  // this call's own plan (the size query may also cover the other reading of B == 1)
  if (!workspace || !aligned16(workspace) || workspace_bytes < plan_forward(dtype, s, opt).total)
    return GDN_ERR_WORKSPACE;

  FwdParams p{};
  p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.h0 = h0; p.cu = cu_seqlens;
  p.o = o; p.hT = hT;
  p.status = static_cast<int*>(workspace);
  p.B = s.B; p.T = s.T; p.Hqk = s.Hqk; p.Hv = s.Hv; p.dk = s.dk; p.dv = s.dv; p.N = s.N;
  p.scale = scale;
  p.qk_l2norm = op.qk_l2norm;
  p.test_stall = op.test_stall;

  if (s.T == 0) return GDN_OK;
  p.status_dev = device_status_word();
  cudaError_t err;
  if (uses_tc(dtype, s)) {
    const FwdPlan f = plan_forward(dtype, s, opt);
    if (workspace_bytes < f.total) return GDN_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    TcPlan plan{};
    plan.kind = kPlanUnits;
    plan.roles = 1;
    const char* what = "";
    // the launch that produces o also writes the chunk start states, when asked
    FwdParams pf = p;
    pf.states = static_cast<__nv_bfloat16*>(save_states);
    if (save_states) {
      pf.chunk_a = reinterpret_cast<float*>(static_cast<uint8_t*>(save_states) + cache_states_bytes(s));
      pf.chunk_p = static_cast<uint8_t*>(save_states) + cache_states_bytes(s) + cache_a_bytes(s);
    }
    int* chunk_off = nullptr;
    if (save_states && s.packed) {           // packed: per-sequence first slot, from cu_seqlens
      chunk_off = reinterpret_cast<int*>(ws + f.off_chunk_off);
      pf.chunk_off = chunk_off;
      if (!f.table) {
        err = launch_cp_plan(p, 1, 0, nullptr, nullptr, nullptr, chunk_off, stream);
        if (err != cudaSuccess) return cuda_fail("chunk offsets", err);
      }
    }
    if (f.kind == kPlanUnits) {
      err = launch_fwd_tc(pf, plan, s.N * s.Hv, stream, &what);
      if (err != cudaSuccess) return cuda_fail(what, err);
      return GDN_OK;
    }
    plan.seg_chunks = f.seg_chunks;
    plan.max_segs = f.max_segs;
    int* first = nullptr;
    if (f.table) {
      plan.table = reinterpret_cast<int2*>(ws + f.off_table);
      plan.table_count = reinterpret_cast<int*>(ws + f.off_count);
      first = reinterpret_cast<int*>(ws + f.off_first);
      err = launch_cp_plan(p, f.seg_chunks, f.max_pairs, const_cast<int2*>(plan.table),
                           const_cast<int*>(plan.table_count), first, chunk_off, stream);
      if (err != cudaSuccess) return cuda_fail("segment table", err);
    }
    if (!f.phased()) {
      plan.kind = kPlanGate;
      err = launch_fwd_tc(pf, plan, f.max_pairs * s.Hv, stream, &what);
      if (err != cudaSuccess) return cuda_fail(what, err);
      return GDN_OK;
    }
    plan.seg_state = reinterpret_cast<float*>(ws + f.off_state);
    plan.seg_trans = reinterpret_cast<float*>(ws + f.off_trans);
    plan.seg_ws = f.fallback ? reinterpret_cast<int*>(ws + f.off_ws) : nullptr;
    if (f.fallback) {                           // every segment's window, before phase 1
      err = launch_cp_probe(p, plan, f.max_pairs * s.Hv, stream, false);
      if (err != cudaSuccess) return cuda_fail("window probe", err);
    }
    plan.kind = kPlanCpP1;
    plan.roles = 2;
    err = launch_fwd_tc(p, plan, f.max_pairs * 2 * s.Hv, stream, &what);
    if (err != cudaSuccess) return cuda_fail(what, err);
    plan.roles = 1;
    err = launch_cp_stitch(p, plan, first, stream);
    if (err != cudaSuccess) return cuda_fail("segment stitch", err);
    plan.kind = kPlanCpP3;
    err = launch_fwd_tc(pf, plan, f.max_pairs * s.Hv, stream, &what);
    if (err != cudaSuccess) return cuda_fail(what, err);
  } else {
    err = launch_fwd_simt(p, dtype == GDN_BF16, stream);
    if (err != cudaSuccess) return cuda_fail("CUDA-core forward", err);
  }
  return GDN_OK;
}

size_t gdn_chunk_states_size(int B, int T, int Hqk, int Hv, int dk, int dv, int num_seqs) {
  Shape s;
  const bool packed = num_seqs > 0 && B == 1;
  if (check_shape(B, T, Hqk, Hv, dk, dv, packed ? num_seqs : 0, packed, s) != GDN_OK) return 0;
  return cache_states_bytes(s) + cache_a_bytes(s) + cache_p_bytes(s);
}

size_t gdn_chunk_bwd_workspace_size(int B, int T, int Hqk, int Hv, int dk, int dv, int num_seqs,
                                    const gdn_options* opt) {
  // B == 1 with num_seqs >= 1 fits both a packed call and a call without cu_seqlens
  Shape s;
  size_t total = kStatusBytes;
  if (check_shape(B, T, Hqk, Hv, dk, dv, 0, false, s) == GDN_OK) total = bwd_workspace_for(s, opt);
  if (num_seqs > 0 && B == 1 && check_shape(B, T, Hqk, Hv, dk, dv, num_seqs, true, s) == GDN_OK)
    total = std::max(total, bwd_workspace_for(s, opt));
  return total;
}

gdn_status gdn_chunk_bwd(gdn_dtype dtype, int B, int T, int Hqk, int Hv, int dk, int dv,
                         const void* q, const void* k, const void* v, const float* g,
                         const void* beta, float scale, const float* h0, const int32_t* cu_seqlens,
                         int num_seqs, const void* dO, const float* dhT, void* dq, void* dk_out,
                         void* dv_out, float* dg, void* dbeta, float* dh0, void* workspace,
                         size_t workspace_bytes, const gdn_options* opt, cudaStream_t stream) {
  if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
  Shape s;
  gdn_status st = check_shape(B, T, Hqk, Hv, dk, dv, num_seqs, cu_seqlens != nullptr, s);
  if (st != GDN_OK) return st;
  gdn_options op;
  st = read_options(opt, op);
  if (st != GDN_OK) return st;
  opt = &op;
  if (T > 0 && (!q || !k || !v || !g || !beta || !dO || !dq || !dk_out || !dv_out || !dg || !dbeta))
    return GDN_ERR_INVALID_ARG;
  const void* cached = op.states;
  const void* ptrs[] = {q, k, v, g, beta, h0, cu_seqlens, dO, dhT, dq, dk_out, dv_out, dg, dbeta, dh0, cached};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (!uses_tc(dtype, s)) {
    // CUDA-core backward (fp32 I/O or head dims 64): no chunk-state cache, no in-kernel q/k
    // normalisation on this path
    if (cached || op.qk_l2norm) return GDN_ERR_UNSUPPORTED;
    const SimtBwdPlan sp = plan_backward_simt(s);
    if (!workspace || !aligned16(workspace) || workspace_bytes < sp.total) return GDN_ERR_WORKSPACE;
    if (s.T == 0) return GDN_OK;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    FwdParams p{};
    p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.h0 = h0; p.cu = cu_seqlens;
    p.status = static_cast<int*>(workspace);
    p.status_dev = device_status_word();
    p.B = s.B; p.T = s.T; p.Hqk = s.Hqk; p.Hv = s.Hv; p.dk = s.dk; p.dv = s.dv; p.N = s.N;
    p.scale = scale;
    const bool grouped = s.Hv != s.Hqk;
    const cudaError_t err = launch_bwd_simt(
        p, dtype == GDN_BF16, dO, dhT, dq, dk_out, grouped ? reinterpret_cast<float*>(ws + sp.off_dq) : nullptr,
        grouped ? reinterpret_cast<float*>(ws + sp.off_dk) : nullptr, dv_out, dg, dbeta, dh0,
        reinterpret_cast<float*>(ws + sp.off_ckpt), reinterpret_cast<float*>(ws + sp.off_tok), sp.grid, stream);
    if (err != cudaSuccess) return cuda_fail("gdn_chunk_bwd (CUDA-core path)", err);
    return GDN_OK;
  }
  if (!state_rows_fit(state_slots(s), s.Hv)) return GDN_ERR_UNSUPPORTED;
  const BwdPlan bp = plan_backward(s, opt);
  if (!workspace || !aligned16(workspace) || workspace_bytes < bp.total) return GDN_ERR_WORKSPACE;
  if (s.T == 0) return GDN_OK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  FwdParams p{};
  p.q = q; p.k = k; p.v = v; p.g = g; p.beta = beta; p.h0 = h0; p.cu = cu_seqlens;
  p.o = nullptr; p.hT = nullptr;
  p.status = static_cast<int*>(workspace);
  p.status_dev = device_status_word();
  p.B = s.B; p.T = s.T; p.Hqk = s.Hqk; p.Hv = s.Hv; p.dk = s.dk; p.dv = s.dv; p.N = s.N;
  p.scale = scale;
  p.qk_l2norm = op.qk_l2norm;
  p.states = cached ? static_cast<__nv_bfloat16*>(const_cast<void*>(cached))
                    : reinterpret_cast<__nv_bfloat16*>(ws + bp.off_states);
  p.chunk_off = s.packed ? reinterpret_cast<int*>(ws + bp.off_chunk_off) : nullptr;
  // per-chunk A, written by the forward pass with the states, read by the chain and the gradients
  uint8_t* cache = static_cast<uint8_t*>(const_cast<void*>(cached));
  p.chunk_a = cached ? reinterpret_cast<float*>(cache + cache_states_bytes(s)) : reinterpret_cast<float*>(ws + bp.off_a);
  p.chunk_p = cached ? cache + cache_states_bytes(s) + cache_a_bytes(s) : ws + bp.off_p;
  __nv_bfloat16* dstates = reinterpret_cast<__nv_bfloat16*>(ws + bp.off_dstates);

  const FwdPlan& f = bp.chain;
  TcPlan plan{};
  plan.kind = kPlanUnits;
  plan.roles = 1;
  plan.seg_chunks = f.seg_chunks;
  plan.max_segs = f.max_segs;
  int items = s.N * s.Hv;
  cudaError_t err;
  const char* what = "";
  int* first = nullptr;                          // packed sequences: first pair index of each sequence
  if (s.packed || f.kind != kPlanUnits) {
    int2* table = f.table ? reinterpret_cast<int2*>(ws + f.off_table) : nullptr;
    int* count = f.table ? reinterpret_cast<int*>(ws + f.off_count) : nullptr;
    first = f.table ? reinterpret_cast<int*>(ws + f.off_first) : nullptr;
    if (s.packed) {
      err = launch_cp_plan(p, f.seg_chunks > 0 ? f.seg_chunks : 1, f.max_pairs, table, count, first,
                           const_cast<int*>(p.chunk_off), stream);
      if (err != cudaSuccess) return cuda_fail("backward plan", err);
    }
    if (f.kind != kPlanUnits) {
      plan.kind = f.phased() ? kPlanCpP3 : kPlanGate;
      plan.table = table;
      plan.table_count = count;
      items = f.max_pairs * s.Hv;
    }
  }
  if (f.phased()) {
    plan.seg_state = reinterpret_cast<float*>(ws + f.off_state);
    plan.seg_trans = reinterpret_cast<float*>(ws + f.off_trans);
    plan.seg_ws = f.fallback ? reinterpret_cast<int*>(ws + f.off_ws) : nullptr;
  }
  TcPlan map_plan = plan;                        // exact stitch, phase 1: two roles per segment
  map_plan.kind = kPlanCpP1;
  map_plan.roles = 2;
  // 1) forward recompute: the bf16 start state of every chunk (unless the caller cached them).
  //    Exact stitch: the segment maps, their chain, then the final pass that stores the states.
  if (!cached) {
    if (f.phased()) {
      FwdParams p1 = p;
      p1.states = nullptr;
      if (f.fallback) {
        err = launch_cp_probe(p, plan, f.max_pairs * s.Hv, stream, false);
        if (err != cudaSuccess) return cuda_fail("window probe", err);
      }
      err = launch_fwd_tc(p1, map_plan, f.max_pairs * 2 * s.Hv, stream, &what);
      if (err != cudaSuccess) return cuda_fail(what, err);
      err = launch_cp_stitch(p, plan, first, stream);
      if (err != cudaSuccess) return cuda_fail("segment stitch", err);
    }
    err = launch_fwd_tc(p, plan, items, stream, &what);
    if (err != cudaSuccess) return cuda_fail(what, err);
  }
  // 2) reverse chain: the state gradient at every chunk end, and dh0. Exact stitch: the mirror of
  //    the forward's, from the sequence end (the segments' maps of the state gradient, their chain
  //    in reverse, then the final pass that stores dS').
  FwdParams pc = p;
  pc.v = dO;
  pc.h0 = dhT;
  pc.hT = dh0;
  pc.states = dstates;
  if (f.phased()) {
    if (f.fallback) {
      err = launch_cp_probe(pc, plan, f.max_pairs * s.Hv, stream, true);
      if (err != cudaSuccess) return cuda_fail("window probe (reverse)", err);
    }
    err = launch_bwd_chain(pc, map_plan, f.max_pairs * 2 * s.Hv, stream, &what);
    if (err != cudaSuccess) return cuda_fail(what, err);
    err = launch_cp_stitch(pc, plan, first, stream, /*reverse=*/true);
    if (err != cudaSuccess) return cuda_fail("segment stitch (reverse)", err);
  }
  err = launch_bwd_chain(pc, plan, items, stream, &what);
  if (err != cudaSuccess) return cuda_fail(what, err);
  // 3) per-chunk gradients
  BwdOut out{};
  out.dq = dq; out.dk = dk_out; out.dv = dv_out; out.dg = dg; out.dbeta = dbeta; out.dO = dO;
  out.dstates = dstates;
  out.chunk_a = p.chunk_a;
  out.chunk_p = p.chunk_p;
  out.qk_partial = bp.grouped ? 1 : 0;
  out.dq_part = bp.grouped ? reinterpret_cast<float*>(ws + bp.off_dq) : nullptr;
  out.dk_part = bp.grouped ? reinterpret_cast<float*>(ws + bp.off_dk) : nullptr;
  err = launch_bwd_grad(p, out, bp.total_chunks, stream, &what);
  if (err != cudaSuccess) return cuda_fail(what, err);
  return GDN_OK;
}

size_t gdn_chunk_host_scratch_size(gdn_host_mode mode, gdn_dtype dtype, int B, int T, int Hqk, int Hv,
                                   int dk, int dv, int num_seqs, const gdn_options* opt) {
  if (mode != GDN_HOST_FWD && mode != GDN_HOST_BWD && mode != GDN_HOST_FWD_BWD) return 0;
  if (dtype != GDN_F32 && dtype != GDN_BF16) return 0;
  gdn_options op;
  if (read_options(opt, op) != GDN_OK) return 0;
  const bool fw = (mode & GDN_HOST_FWD) != 0, bw = (mode & GDN_HOST_BWD) != 0;
  Shape s;
  size_t total = 0;
  if (check_shape(B, T, Hqk, Hv, dk, dv, 0, false, s) == GDN_OK) total = host_layout(dtype, s, fw, bw, op).total;
  if (num_seqs > 0 && B == 1 && check_shape(B, T, Hqk, Hv, dk, dv, num_seqs, true, s) == GDN_OK)
    total = std::max(total, host_layout(dtype, s, fw, bw, op).total);
  return total;
}

gdn_status gdn_chunk_host(gdn_host_mode mode, gdn_dtype dtype, int B, int T, int Hqk, int Hv, int dk, int dv,
                          const void* q, const void* k, const void* v, const float* g, const void* beta,
                          float scale, const float* h0, const int32_t* cu_seqlens, int num_seqs,
                          const void* dO, const float* dhT, void* o, float* hT, void* dq, void* dk_out,
                          void* dv_out, float* dg, void* dbeta, float* dh0, void* scratch, size_t scratch_bytes,
                          const gdn_options* opt, cudaStream_t stream, cudaStream_t h2d_stream,
                          cudaStream_t d2h_stream) {
  // every check that the device calls below make, before the first copy is enqueued
  if (mode != GDN_HOST_FWD && mode != GDN_HOST_BWD && mode != GDN_HOST_FWD_BWD) return GDN_ERR_INVALID_ARG;
  if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
  Shape s;
  gdn_status st = check_shape(B, T, Hqk, Hv, dk, dv, num_seqs, cu_seqlens != nullptr, s);
  if (st != GDN_OK) return st;
  gdn_options op;
  st = read_options(opt, op);
  if (st != GDN_OK) return st;
  if (op.states) return GDN_ERR_INVALID_ARG;       // the call keeps its own cache in the scratch
  const bool fw = (mode & GDN_HOST_FWD) != 0, bw = (mode & GDN_HOST_BWD) != 0;
  if (T > 0) {
    if (!q || !k || !v || !g || !beta) return GDN_ERR_INVALID_ARG;
    if (fw && !o) return GDN_ERR_INVALID_ARG;
    if (bw && (!dO || !dq || !dk_out || !dv_out || !dg || !dbeta)) return GDN_ERR_INVALID_ARG;
  }
  if (bw && uses_tc(dtype, s) && !state_rows_fit(state_slots(s), s.Hv)) return GDN_ERR_UNSUPPORTED;
  if (op.qk_l2norm && !uses_tc(dtype, s)) return GDN_ERR_UNSUPPORTED;
  const HostLayout L = host_layout(dtype, s, fw, bw, op);
  if (!scratch || (reinterpret_cast<uintptr_t>(scratch) & 255u) != 0 || scratch_bytes < L.total)
    return GDN_ERR_WORKSPACE;
  if (s.T == 0) return GDN_OK;

  HostEvents* ev = nullptr;
  st = host_events(scratch, ev);
  if (st != GDN_OK) return st;
  HostEventsHold hold{ev};
  uint8_t* sb = static_cast<uint8_t*>(scratch);
  const cudaStream_t hs = h2d_stream ? h2d_stream : stream, ds = d2h_stream ? d2h_stream : stream;
  cudaError_t err = cudaSuccess;
  auto h2d = [&](size_t off, const void* src, size_t n) {
    if (src && n && err == cudaSuccess) err = cudaMemcpyAsync(sb + off, src, n, cudaMemcpyHostToDevice, hs);
  };
  auto d2h = [&](void* dst, size_t off, size_t n) {
    if (dst && n && err == cudaSuccess) err = cudaMemcpyAsync(dst, sb + off, n, cudaMemcpyDeviceToHost, ds);
  };
  auto record = [&](cudaEvent_t e, cudaStream_t on) {
    if (err == cudaSuccess) err = cudaEventRecord(e, on);
  };
  auto wait = [&](cudaStream_t on, cudaEvent_t e) {
    if (err == cudaSuccess) err = cudaStreamWaitEvent(on, e, 0);
  };
  auto dev = [&](size_t off, const void* host_ptr) -> void* { return host_ptr ? sb + off : nullptr; };

  // inputs in, once the previous call on this scratch has finished reading them; the forward's
  // arrays first, so that it can start while dO, dhT are still coming in
  if (ev->used) wait(hs, ev->compute_done);
  h2d(L.q, q, L.n_qk);
  h2d(L.k, k, L.n_qk);
  h2d(L.v, v, L.n_v);
  h2d(L.g, g, L.n_g);
  h2d(L.beta, beta, L.n_beta);
  h2d(L.h0, h0, L.n_h);
  h2d(L.cu, cu_seqlens, s.packed ? L.n_cu : 0);
  record(ev->in_fwd, hs);
  if (bw) {
    h2d(L.dO, dO, L.n_v);
    h2d(L.dhT, dhT, L.n_h);
    record(ev->in_bwd, hs);
  }
  // the kernels, once the previous call's output copies from this scratch are done
  if (ev->used) wait(stream, ev->out_done);
  wait(stream, ev->in_fwd);
  if (err != cudaSuccess) return cuda_fail("gdn_chunk_host: enqueue", err);
  const float* d_h0 = static_cast<const float*>(dev(L.h0, h0));
  const int32_t* d_cu = static_cast<const int32_t*>(dev(L.cu, cu_seqlens));
  gdn_options od = op;
  const bool cache = fw && bw && uses_tc(dtype, s);   // otherwise the backward recomputes its forward pass
  if (fw) {
    od.states = cache ? sb + L.states : nullptr;
    st = gdn_chunk_fwd(dtype, B, T, Hqk, Hv, dk, dv, sb + L.q, sb + L.k, sb + L.v,
                       reinterpret_cast<const float*>(sb + L.g), sb + L.beta, scale, d_h0, d_cu, num_seqs,
                       sb + L.o, static_cast<float*>(dev(L.hT, hT)), sb + L.ws_f, L.ws_f_bytes, &od, stream);
    if (st != GDN_OK) return st;
    record(ev->fwd_done, stream);
    wait(ds, ev->fwd_done);                        // o, hT go back while the backward runs
    d2h(o, L.o, L.n_v);
    d2h(hT, L.hT, L.n_h);
  }
  if (bw) {
    wait(stream, ev->in_bwd);
    if (err != cudaSuccess) return cuda_fail("gdn_chunk_host: enqueue", err);
    od.states = cache ? sb + L.states : nullptr;
    st = gdn_chunk_bwd(dtype, B, T, Hqk, Hv, dk, dv, sb + L.q, sb + L.k, sb + L.v,
                       reinterpret_cast<const float*>(sb + L.g), sb + L.beta, scale, d_h0, d_cu, num_seqs,
                       sb + L.dO, static_cast<const float*>(dev(L.dhT, dhT)), sb + L.dq, sb + L.dk, sb + L.dv,
                       reinterpret_cast<float*>(sb + L.dg), sb + L.dbeta, static_cast<float*>(dev(L.dh0, dh0)),
                       sb + L.ws_b, L.ws_b_bytes, &od, stream);
    if (st != GDN_OK) return st;
  }
  record(ev->compute_done, stream);
  if (bw) {
    wait(ds, ev->compute_done);
    d2h(dq, L.dq, L.n_qk);
    d2h(dk_out, L.dk, L.n_qk);
    d2h(dv_out, L.dv, L.n_v);
    d2h(dg, L.dg, L.n_g);
    d2h(dbeta, L.dbeta, L.n_beta);
    d2h(dh0, L.dh0, L.n_h);
  }
  record(ev->out_done, ds);
  if (err != cudaSuccess) return cuda_fail("gdn_chunk_host: enqueue", err);
  ev->used = true;
  return GDN_OK;
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
  return device_code_status(code);
}

gdn_status gdn_check_device_error(cudaStream_t stream) {
  cudaError_t err = cudaStreamSynchronize(stream);
  if (err != cudaSuccess) return cuda_fail("gdn_check_device_error: stream", err);
  int code = 0;
  err = cudaMemcpyFromSymbol(&code, g_device_status, sizeof(int));
  if (err != cudaSuccess) return cuda_fail("gdn_check_device_error: read", err);
  if (code != 0) {
    const int zero = 0;
    err = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
    if (err != cudaSuccess) return cuda_fail("gdn_check_device_error: clear", err);
  }
  return device_code_status(code);
}

}  // extern "C"
