// Tensor-core (tcgen05 / TMEM / TMA) forward of the GDN chunked prefill for bf16 I/O,
// dk = dv = 128, 64-token chunks. One CTA runs the whole chunk sequence of one work
// item (a (sequence, v-head) unit, or one segment of it under context parallelism).
//
// The recurrence is carried as S = h^T (dv x dk, fp32, in TMEM) so that every
// tensor-core product has M = 128 rows = the dv rows of S (or the dk rows of W^T, or the
// 128 stacked K;Q token rows of the Gram product). Per chunk (gam = chunk-local inclusive
// cumsum of g, E_ij = exp(gam_i - gam_j)):
//
//   prep warps (state independent, overlap the previous chunk's chain):
//     G  = [K;Q] K^T                               tcgen05, M=128 N=64 K=128
//     L  = strict_lower(diag(beta) KK^T * E) (fp16),  A = (I + L)^-1 (fp32): 16 x 16 diagonal
//          blocks by substitution (CUDA cores), the blocks below by 2 x 2 blocking on m16n8k16 f16
//          products;  P = lower_incl(QK^T * E) -> bf16
//   epilogue warps, handing over to the chunk (in what would otherwise be a wait for the prep):
//     Q <- diag(exp(gam)) Q  (Q~);  A2 = A diag(beta), B2 = A diag(beta exp(gam)) -> bf16
//     U^T = V^T A2^T   into the chunk's Delta accumulator          tcgen05, M=128 N=64 K=64
//     W   = B2 K       -> -W in bf16 over the V tile (token rows)   tcgen05, M=64 N=128 K=64
//   epilogue warps (the sequential chain, two tensor-core round trips per chunk):
//     (a) [D_Q | Delta^T] += S_bf16 [Q~ ; -W]^T  (D_Q from zero, Delta^T onto U^T)
//                                                                  tcgen05, M=128 N=128 K=128
//     (b) Delta^T -> bf16, Delta~^T = Delta^T diag(exp(gam_n - gam)) -> bf16
//     (c) D_Q += Delta^T P^T;  S += Delta~^T K   (K read MN-major from the TMA tile)
//     (d) S -> bf16 for the next chunk's products;  O = scale * D_Q
// i.e. Delta = U - W h with U = A diag(beta) V and W = A diag(beta e^gam) K,
// O = scale[diag(e^gam) Q h + (QK^T*E*M) Delta], h' = e^gam_n h + (diag(e^(gam_n-gam)) K)^T Delta:
// the WY/UT chunkwise form of the gated delta rule ("FlashQLA resource", section 3: fused
// warp-specialised kernels that overlap data movement, tensor-core and CUDA-core work).
#include <cudaTypedefs.h>

#include "gdn_chunk_prep.cuh"
#include "gdn_common.cuh"
#include "gdn_tc.cuh"
#include "tc_ptx.cuh"

namespace gdn {
using namespace tc;

namespace {

constexpr int kThreads = 512;             // 16 warps
constexpr int kEpiWarp0 = 8;              // warps 0-7: prep (TMEM lane quadrant w % 4, column half w / 4)
                                          // warps 8-15: epilogue (same split); the epilogue's first
                                          // thread also issues the TMA loads and the chain MMAs
constexpr int kNumPrep = 256, kNumEpi = 256;
constexpr int kBarPrep = 1, kBarEpi = 2;  // named barrier ids
constexpr int kBarScalars = 3;            // prep warps 0-1: the chunk's g, beta and decay scalars
constexpr int kGramIssuer = 224;          // lane 0 of prep warp 7 (no part in the scalar scan)

// shared memory layout (bytes from a 1024-aligned base)
constexpr uint32_t kStageBytes = 48u * 1024u;   // [K0 Q0 V0 | K1 Q1 V1], 8KB 128B-swizzled sub-tiles
constexpr uint32_t kHalf = 24u * 1024u;         // feature columns 64..127 of K, Q, V
constexpr uint32_t kOffQ = 8u * 1024u;          // within a half
constexpr uint32_t kOffV = 16u * 1024u;         // within a half: V, then -W (token rows)
constexpr uint32_t kOffA2 = 96u * 1024u;        // 8KB      A diag(beta), bf16, SW128 rows
constexpr uint32_t kOffB2 = 104u * 1024u;       // 8KB      A diag(beta exp(gam)), bf16
constexpr uint32_t kOffP = 112u * 1024u;        // 2 x 8KB  masked decayed QK^T, bf16
constexpr uint32_t kOffSb = 128u * 1024u;       // 32KB     S in bf16 (two 64-col sub-tiles)
constexpr uint32_t kOffYt = 160u * 1024u;       // 16KB     Delta^T, bf16 [dv][token]
constexpr uint32_t kOffDt = 176u * 1024u;       // 16KB     Delta~^T, then O staging (two swizzled 64-column halves)
constexpr uint32_t kOffLf = 192u * 1024u;       // fp16 [64][kLdh] L, diagonal blocks inverted in place
constexpr uint32_t kOffAst = kOffLf + 64u * kLdh * 2u;   // 16KB  A in fp32 (stored-A layout; bulk-copied for the backward)
constexpr uint32_t kOffSmall = kOffAst + 16384u;

struct Small {
  ChunkScalars cs;
  float wsum[16];         // warm-up window search: per-warp partial sums
  uint64_t full_k[2], full_qv[2], prep_full[2], gdone, wdone, mma_done;
  uint64_t dd_free[2];    // by stage: the chain has read the chunk's W and its scalars (step (c))
  uint64_t dec_ready[2];  // by stage: the chunk's decay scalars written and its Gram product done
  uint64_t a_free;        // the chain has read the chunk's fp32 A (the prep may write the next one)
  uint64_t stall;         // testing only: a barrier that nothing completes
  uint32_t tmem_base;
  int abort_flag;
};
constexpr uint32_t kSmemBytes = kOffSmall + sizeof(Small);
static_assert(kSmemBytes <= 232448, "dynamic shared memory above the 227 KB a block can opt into");
constexpr long long kStallCycles = 1LL << 21;   // ~1 ms: limit of the testing hook's wait

// TMEM columns (fp32, 128 lanes)
constexpr uint32_t kColGW = 0;      // 2 x 128 by chunk parity: [K;Q] K^T (64 cols); then
                                    //   W (M=64 layout: row m in lane m%16 + 32(m/16), 128 cols)
constexpr uint32_t kColPair = 256;  // 128: [D_Q | Delta^T]
                                    //   D_Q = S Q~^T + Delta^T P^T,  Delta^T = U^T - S W^T
constexpr uint32_t kColDd = kColPair + 64;
constexpr uint32_t kColS = 384;     // 128: the fp32 state S (dv x dk), updated in place
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kId64 = idesc_bf16(128, 64, false, false);     // A, B K-major
constexpr uint32_t kId128 = idesc_bf16(128, 128, false, false);   // A, B K-major
constexpr uint32_t kIdU = idesc_bf16(128, 64, true, false);       // A MN-major
constexpr uint32_t kIdW = idesc_bf16(64, 128, false, true);       // B MN-major, M = 64
constexpr uint32_t kIdE2 = idesc_bf16(128, 128, false, true);     // B MN-major


}  // namespace

// kNorm: q and k rows are L2-normalised in the kernel (their inverse norms folded into the
// per-token factors; see ChunkScalars).
template <bool kNorm>
__global__ void __launch_bounds__(kThreads, 1)
gdn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_s,
                  const __grid_constant__ CUtensorMap tm_o, const FwdParams p, const TcPlan plan) {
  // Dynamic shared memory starts at the (1024-aligned) base of the CTA's window: the
  // kernel has no static shared variables. Used directly so every access stays a
  // shared-space access.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  Small* ss = reinterpret_cast<Small*>(sm + kOffSmall);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if ((smem_u32(sm) & 1023u) != 0) {                     // 128B-swizzled tiles need 1024B alignment
    if (threadIdx.x == 0) report_error(p, kDevMisaligned);
    return;
  }
  if (plan.seg_ws != nullptr && plan.kind == kPlanCpP1) {
    // exact fallback, phase 1: item = (pi * 2 + role) * Hv + j. When the successor's window closes
    // (the probe's record, read before anything else) no map is needed: leave at once.
    const int j = blockIdx.x % p.Hv, pi = blockIdx.x / (2 * p.Hv);
    if ((pi + 1) * 2 * p.Hv < (int)gridDim.x && plan.seg_ws[(size_t)(pi + 1) * p.Hv + j] >= 0) return;
  }
  WorkItem it;
  if (!get_work_item(p, plan, blockIdx.x, it)) return;   // uniform over the CTA
  const __nv_bfloat16* beta = static_cast<const __nv_bfloat16*>(p.beta);

  // First token this CTA processes (ws), decided before any setup so that a phase-1 CTA with
  // nothing to do leaves at once. Gate-driven warm-up (context parallelism): a segment that starts
  // inside a sequence begins from a zero state at the start of a window of earlier chunks whose
  // transition has spectral norm <= prod_t exp(g_t) max(1, |1 - beta_t |k_t|^2|) <= 2^-64: the
  // state it drops is then below fp32 resolution. Each token's factor is the exact norm of
  // exp(g)(I - beta k k^T); the window walks back chunk by chunk (at most kMaxWarm chunks).
  //   gate-driven plan: without such a window the segment starts at the sequence start with h0.
  //   with the exact stitch as fallback (plan.seg_ws, every segment's window recorded by the
  //     probe kernel): in phase 1, when the successor's window closes it needs no map and the CTA
  //     leaves; otherwise the segment's map is computed, or, when the segment's own window closes,
  //     its end state straight from that window (role 0). Phase 3 starts from the window or from
  //     the stitched state.
  int ws = it.s;
  if (it.gate) {
    if (it.s > it.seq_s) {
      const int w = gate_window_start(p, it, it.s, ss->wsum);
      ws = w >= 0 ? w : it.seq_s;
    }
  } else if (plan.seg_ws != nullptr && plan.kind == kPlanCpP1) {
    if (plan.seg_ws[(size_t)(it.pi + 1) * p.Hv + it.j] >= 0) return;
    if (it.seg > 0) {
      const int w0 = plan.seg_ws[(size_t)it.pi * p.Hv + it.j];
      if (w0 >= 0) {
        if (it.role == 1) return;
        ws = w0;
      }
    }
  } else if (plan.seg_ws != nullptr && plan.kind == kPlanCpP3 && it.seg > 0) {
    const int w = plan.seg_ws[(size_t)it.pi * p.Hv + it.j];
    if (w >= 0) ws = w;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ss->full_k[s], 1);
      mbar_init(&ss->full_qv[s], 1);
      mbar_init(&ss->prep_full[s], 1);
      mbar_init(&ss->dec_ready[s], 1);
    }
    mbar_init(&ss->gdone, 1);
    mbar_init(&ss->wdone, 1);
    mbar_init(&ss->dd_free[0], 1);
    mbar_init(&ss->dd_free[1], 1);
    mbar_init(&ss->a_free, 1);
    mbar_init(&ss->mma_done, 1);
    mbar_init(&ss->stall, 1);
    ss->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ss->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == kEpiWarp0 * 32) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // Testing hook: one thread waits on a barrier that nothing completes. The wait gives up
  // after ~1 ms and the CTA reports a timed-out wait; the chunk work below then runs as usual
  // (its own waits keep their normal limit), so the context stays usable.
  if (p.test_stall) {
    if (threadIdx.x == 0) {
      volatile int stall_flag = 0;
      if (!mbar_wait_limit(&ss->stall, 0, &stall_flag, kStallCycles)) report_error(p, kDevTimeout);
    }
    __syncthreads();
  }

  const int nchunks = (it.e - ws + kChunk - 1) / kChunk;
  const bool from_seq_start = (ws == it.seq_s);
  const int init_mode = (ws == it.s) ? it.init_mode : (from_seq_start && p.h0 ? (int)kInitPtr : (int)kInitZero);
  const float* init_ptr = (ws == it.s) ? it.init : p.h0 + ((size_t)it.n * p.Hv + it.j) * (size_t)(128 * 128);

  const uint32_t tmem = ss->tmem_base;
  volatile int* abort_flag = &ss->abort_flag;
  const uint32_t sbase = smem_u32(sm);

  // TMA loads of chunk c into stage c % 2, issued by the epilogue's first thread: chunks 0
  // and 1 at the start; for chunk c + 2, the Q and V tiles as soon as chunk c's state product
  // has read Q~ and -W, the K tiles once its update product has read K.
  auto load_k = [&](int c) {
    const int s = c & 1;
    const int row = it.b * p.T + ws + c * kChunk;
    uint8_t* st = sm + s * kStageBytes;
    mbar_arrive_expect_tx(&ss->full_k[s], 16u * 1024u);
    tma_load_3d(st, &tm_k, &ss->full_k[s], 0, it.hq, row);
    tma_load_3d(st + kHalf, &tm_k, &ss->full_k[s], 64, it.hq, row);
  };
  auto load_qv = [&](int c) {
    const int s = c & 1;
    const int row = it.b * p.T + ws + c * kChunk;
    uint8_t* st = sm + s * kStageBytes;
    mbar_arrive_expect_tx(&ss->full_qv[s], it.zero_v ? 16u * 1024u : 32u * 1024u);
    tma_load_3d(st + kOffQ, &tm_q, &ss->full_qv[s], 0, it.hq, row);
    tma_load_3d(st + kHalf + kOffQ, &tm_q, &ss->full_qv[s], 64, it.hq, row);
    if (!it.zero_v) {
      tma_load_3d(st + kOffV, &tm_v, &ss->full_qv[s], 0, it.j, row);
      tma_load_3d(st + kHalf + kOffV, &tm_v, &ss->full_qv[s], 64, it.j, row);
    }
  };

  // Every role keeps executing its loop (and its named barriers) after an aborted
  // wait, with the work skipped: a role never leaves its peers stuck at a barrier.
  if (warp < kEpiWarp0) {
    // ------------------------------------------------------------ prep (8 warps)
    const int pt = threadIdx.x;            // 0..255
    PrepCtx pc{sbase, reinterpret_cast<float*>(sm + kOffLf), &ss->cs, tmem, kColGW, pt, warp, lane, kBarPrep};
    bool ok = true;
    // g, beta of a chunk (0 past the sequence end), loaded one chunk ahead
    auto load_gb = [&](int c, float& gv, float& bv) {
      const int t0 = ws + c * kChunk;
      gv = 0.f;
      bv = 0.f;
      if (pt < kChunk && t0 + pt < it.e) {
        const size_t gi = (size_t)(it.b * p.T + t0 + pt) * p.Hv + it.j;
        gv = p.g[gi];
        bv = __bfloat162float(beta[gi]);
      }
    };
    // Start of chunk c: wait for its tiles, clear rows past the sequence end, issue
    // G = [K;Q] K^T into G/W buffer c % 2 and form the chunk's decay scalars.
    auto chunk_start = [&](int c, float gv, float bv) {
      const int s = c & 1;
      const int nv = min(kChunk, it.e - (ws + c * kChunk));
      // chunk c - 2 (same slot) is done with: the chain has read its W and its scalars (each stage's
      // barrier completes once per two chunks; chunk c's own phase cannot complete before its prep)
      if (c >= 2) {
        ok = ok && mbar_wait(&ss->dd_free[s], ((c - 2) >> 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
      }
      uint8_t* st = sm + s * kStageBytes;
      const uint32_t st_addr = sbase + s * kStageBytes;
      ok = ok && mbar_wait(&ss->full_k[s], (c >> 1) & 1, abort_flag);
      ok = ok && mbar_wait(&ss->full_qv[s], (c >> 1) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      // full chunk: the Gram product can start at once, issued by warp 7 while warps 0-1 form the
      // scalars (a partial chunk waits for its zeroed rows)
      if (nv == kChunk && pt == kGramIssuer && ok) issue_gram(tmem + kColGW + 128u * s, st_addr, &ss->gdone, kHalf);
      prep_store_gb(pc, s, gv, bv);
      if (nv < kChunk) {
        // rows past the sequence end hold the next sequence's tokens: clear them
        const int tiles = it.zero_v ? 4 : 6;
        for (int idx = pt; idx < (kChunk - nv) * tiles * 8; idx += kNumPrep) {
          const int r = nv + idx / (tiles * 8), rem = idx % (tiles * 8), tile = rem / 8, ch = rem % 8;
          // tiles 0..3: K0 Q0 K1 Q1; 4, 5: V0 V1
          const uint32_t toff = tile < 4 ? (tile >> 1) * kHalf + (tile & 1) * kOffQ : (tile - 4) * kHalf + kOffV;
          *reinterpret_cast<uint4*>(st + toff + r * 128u + ch * 16u) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        named_bar_sync(kBarPrep, kNumPrep);
        if (pt == 0 && ok) issue_gram(tmem + kColGW + 128u * s, st_addr, &ss->gdone, kHalf);
      } else if (pt < kChunk) {
        named_bar_sync(kBarScalars, kChunk);      // g, beta of warps 0-1 -> the scan (warp 0)
      }
      if (kNorm) row_inv_norms(st, st + kHalf, st + kOffQ, st + kHalf + kOffQ, ss->cs.rk[s], ss->cs.rq[s], pt);
      prep_scan(pc, s);
      // the bulk copies of earlier P tiles have read their slots (this chunk's masks rewrite one)
      if (pt == 0) bulk_wait_read();
      named_bar_sync(kBarPrep, kNumPrep);
      prep_decays<kNorm>(pc, s, nv);
      // warps 0-1 wrote the decay scalars; thread 0 publishes them to the chain (dec_ready) once the
      // Gram product is also done, at the top of this chunk's prep iteration
      if (pt < kChunk) named_bar_sync(kBarScalars, kChunk);
    };
    // Iteration c runs chunk c's prep, then chunk c + 1's start; iteration -1 only the first
    // start (each phase has one call site: the kernel's code stays small for the instruction cache)
    for (int c = -1; c < nchunks; ++c) {
      float gv1 = 0.f, bv1 = 0.f;
      if (c + 1 < nchunks) load_gb(c + 1, gv1, bv1);
      if (c >= 0) {
      const int s = c & 1;
      const uint32_t gw_col = kColGW + 128u * s;
      ok = ok && mbar_wait(&ss->gdone, c & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      // the Gram product has read Q and the decays are written: the chain may scale Q (Q~)
      if (pt == 0 && ok) mbar_arrive(&ss->dec_ready[s]);
      pc.colG = gw_col;
      prep_masks<true, kNorm>(pc, s, sbase + kOffP + s * 8192u, 1.f, ok);
      // A = (I + L)^-1 in fp32 into the A staging buffer (also the backward's copy): diagonal
      // blocks on warps 0-3 while warps 4-7 clear A's upper blocks; then the blocked inverse below
      // the diagonal (Q~ is formed by the chain warps, see dec_ready)
      float* af = reinterpret_cast<float*>(sm + kOffAst);
      if (c > 0) {                                     // the chain has read chunk c - 1's A
        ok = ok && mbar_wait(&ss->a_free, (c - 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (warp < 4) prep_diag_inverse_h(pc, af);
      else af_zero_upper(af, pt - 128, 128);
      named_bar_sync(kBarPrep, kNumPrep);
      prep_inverse_blocked(pc, af);
      // A complete in fp32 (the chain forms A2, B2 from it and issues the U^T, W products)
      fence_proxy_async_smem();
      named_bar_sync(kBarPrep, kNumPrep);
      if (pt == 0 && p.states != nullptr && p.chunk_p != nullptr && ws + c * kChunk >= it.s && ok) {
        // P for the backward: one bulk copy of the operand tile (fenced above); its reads are
        // waited for before the tile's slot is rewritten two chunks later
        const size_t slot = chunk_slot(p, it.n, (ws + c * kChunk - it.seq_s) / kChunk) * p.Hv + it.j;
        bulk_store(p.chunk_p + slot * 8192, sbase + kOffP + s * 8192u, 8192u);
        if (p.chunk_a != nullptr) bulk_store(p.chunk_a + slot * (kChunk * kChunk), sbase + kOffAst, 16384u);
        bulk_commit();
      }
      tc_fence_before();
      if (pt == 0 && ok) mbar_arrive(&ss->prep_full[s]);
      }
      // the next chunk's start (its Gram product goes to the other G/W buffer)
      if (c + 1 < nchunks) chunk_start(c + 1, gv1, bv1);
    }
    if (pt == 0) bulk_wait_all();
  } else {
    // ------------------------------------------------------------ epilogue: the state chain
    const int et = threadIdx.x - kEpiWarp0 * 32;  // 0..255
    const int ew = et >> 5;
    const int qd = ew & 3, hh = ew >> 2;
    const int r = 32 * qd + lane;                 // dv row of S (= TMEM lane)
    const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
    const uint32_t s_addr = tmem + lane_base + kColS + hh * 64;
    // for the A2 / B2 formation, which takes the group's thread index
    const PrepCtx ec{sbase, reinterpret_cast<float*>(sm + kOffLf), &ss->cs, tmem, kColGW, et, ew, lane, kBarEpi};   // this thread's 64 columns of S
    // initial state -> TMEM (fp32) and Sb (bf16)
    auto write_sb = [&](const float* v, int half32) {
      const uint32_t base = sbase + kOffSb + hh * 16384u;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const int ch = half32 * 4 + c4;
        st_shared_v4(base + sw128(r, ch), pack_bf16(v[c4 * 8 + 0], v[c4 * 8 + 1]),
                     pack_bf16(v[c4 * 8 + 2], v[c4 * 8 + 3]), pack_bf16(v[c4 * 8 + 4], v[c4 * 8 + 5]),
                     pack_bf16(v[c4 * 8 + 6], v[c4 * 8 + 7]));
      }
    };
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      float v[32];
#pragma unroll
      for (int d = 0; d < 32; ++d) {
        const int col = hh * 64 + h2 * 32 + d;
        if (init_mode == kInitPtr) v[d] = init_ptr[(size_t)col * 128 + r];
        else if (init_mode == kInitIdentity) v[d] = (col == r) ? 1.f : 0.f;
        else v[d] = 0.f;
      }
      tmem_st32_sync(s_addr + h2 * 32, v);
      write_sb(v, h2);
    }
    {
      float z[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) z[u] = 0.f;
      tmem_st32_sync(tmem + lane_base + kColPair + hh * 32, z);          // D_Q starts at 0
    }
    fence_proxy_async_smem();
    tc_fence_before();
    named_bar_sync(kBarEpi, kNumEpi);
    uint32_t mph = 0;
    // (a) [D_Q | Delta^T] += S_bf16 [Q~ ; -W]^T: B = rows Q~ then -W, adjacent in each half of
    //     the stage. D_Q was zeroed after its last read; Delta^T holds the prep's U^T (or 0).
    auto issue_a = [&](int c) {
      tc_fence_after();
      const uint32_t a0 = sbase + kOffSb, b0 = sbase + (c & 1) * kStageBytes + kOffQ;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_f16(tmem + kColPair, sdesc_sw128(a0 + (ks >> 2) * 16384u + (ks & 3) * 32u, 16, 1024),
                 sdesc_sw128(b0 + (ks >> 2) * kHalf + (ks & 3) * 32u, 16, 1024), kId128, 1);
      umma_commit(&ss->mma_done);
    };
    // S <- exp(gam_n) S in TMEM (before the chunk's update accumulates onto it)
    auto prescale = [&](int s) {
      const float egn = ss->cs.egn[s];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        float v[32];
        tmem_ld32_sync(s_addr + h2 * 32, v);
#pragma unroll
        for (int d = 0; d < 32; ++d) v[d] *= egn;
        tmem_st32_sync(s_addr + h2 * 32, v);
      }
    };
    bool ok = true;
    int loaded_k = 0, loaded_qv = 0;              // chunks whose K / Q,V loads were issued (et == 0)
    // Chunk c's W (the prep's product, M = 64 layout in G/W buffer c % 2) -> -W in bf16 token
    // rows over the stage's V tile, which the U^T product has consumed: warp (qd, hh) holds
    // tokens 16 qd + lane (lanes 0..15) at features 64 hh .. 64 hh + 63. Ends with the
    // epilogue barrier.
    auto store_w = [&](int c) {
      ok = ok && mbar_wait(&ss->wdone, c & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      float v[32], v2[32];
      const uint32_t gw = tmem + lane_base + kColGW + 128u * (c & 1) + 64 * hh;
      if (ok) {
        tmem_ld32_sync(gw, v);
        tmem_ld32_sync(gw + 32, v2);
      } else {
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = v2[u] = 0.f;
      }
      if (lane < 16) {
        const int jr = 16 * qd + lane;
        const uint32_t wb = sbase + (c & 1) * kStageBytes + hh * kHalf + kOffV;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          st_shared_v4(wb + sw128(jr, c4), pack_bf16(-v[8 * c4], -v[8 * c4 + 1]),
                       pack_bf16(-v[8 * c4 + 2], -v[8 * c4 + 3]), pack_bf16(-v[8 * c4 + 4], -v[8 * c4 + 5]),
                       pack_bf16(-v[8 * c4 + 6], -v[8 * c4 + 7]));
          st_shared_v4(wb + sw128(jr, 4 + c4), pack_bf16(-v2[8 * c4], -v2[8 * c4 + 1]),
                       pack_bf16(-v2[8 * c4 + 2], -v2[8 * c4 + 3]), pack_bf16(-v2[8 * c4 + 4], -v2[8 * c4 + 5]),
                       pack_bf16(-v2[8 * c4 + 6], -v2[8 * c4 + 7]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarEpi, kNumEpi);
    };
    if (et == 0) {
      for (; loaded_k < 2 && loaded_k < nchunks; ++loaded_k) {
        load_k(loaded_k);
        load_qv(loaded_k);
      }
      loaded_qv = loaded_k;
    }
    auto wait_mma = [&]() {
      ok = ok && mbar_wait(&ss->mma_done, mph, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      mph ^= 1;
      tc_fence_after();
    };
    // Iteration c runs chunk c's chain, then hands over to chunk c + 1 (-W, its first product, the
    // prescale); iteration -1 only the first hand-over (one call site per phase: the kernel's code
    // stays small for the instruction cache)
    for (int c = -1; c < nchunks; ++c) {
      const int s = c & 1;
      const int t0 = ws + c * kChunk;
      bool write_o = false, o_tma = false;
      int nv = 0;
      if (c >= 0) {
      nv = ss->cs.nv[s];                            // read before step (c) releases the chunk's scalars
      wait_mma();
      if (et == 0 && ok && c + 2 < nchunks) {     // Q~ and -W of stage s are consumed
        load_qv(c + 2);
        loaded_qv = c + 3;
      }
      if (et == 0 && p.states != nullptr && t0 >= it.s && ok) {
        // backward support: this chunk's start state (the bf16 copy its products use), two TMA
        // tile stores from the swizzled copy; waited for (reads) before the copy is rewritten
        const int srow = (int)((chunk_slot(p, it.n, (t0 - it.seq_s) / kChunk) * p.Hv + it.j) * 128);
        tma_store_3d(&tm_s, sbase + kOffSb, 0, 0, srow);
        tma_store_3d(&tm_s, sbase + kOffSb + 16384u, 64, 0, srow);
        bulk_commit();
      }
      // (b) Delta^T and Delta~^T = Delta^T diag(exp(gam_n - gam)) -> bf16
      {
        float dd[32];
        if (ok) tmem_ld32_sync(tmem + lane_base + kColDd + hh * 32, dd);
        else {
#pragma unroll
          for (int u = 0; u < 32; ++u) dd[u] = 0.f;
        }
        const float* egd = ss->cs.egd[s];
        uint32_t w[16], x[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int j0 = hh * 32 + 2 * u;
          w[u] = pack_bf16(dd[2 * u], dd[2 * u + 1]);
          x[u] = pack_bf16(dd[2 * u] * egd[j0], dd[2 * u + 1] * egd[j0 + 1]);
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          st_shared_v4(sbase + kOffYt + sw128(r, hh * 4 + c4), w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
          st_shared_v4(sbase + kOffDt + sw128(r, hh * 4 + c4), x[4 * c4], x[4 * c4 + 1], x[4 * c4 + 2], x[4 * c4 + 3]);
        }
      }
      if (et == 0) bulk_wait_read();                // Sb is rewritten after this barrier
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarEpi, kNumEpi);
      // (c) D_Q += Delta^T P^T;  S += Delta~^T K   (S was pre-scaled by exp(gam_n))
      if (et == 0 && ok) {
        mbar_arrive(&ss->dd_free[s]);             // chunk c's scalars and W are read: the prep may reuse the slot
        tc_fence_after();
        const uint32_t ya = sbase + kOffYt, pb = sbase + kOffP + s * 8192u;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_f16(tmem + kColPair, sdesc_sw128(ya + ks * 32, 16, 1024),
                   sdesc_sw128(pb + ks * 32, 16, 1024), kId64, 1);
        const uint32_t da = sbase + kOffDt, kb = sbase + s * kStageBytes;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_f16(tmem + kColS, sdesc_sw128(da + ks * 32, 16, 1024), sdesc_sw128(kb + ks * 2048, kHalf, 1024),
                   kIdE2, 1);
        umma_commit(&ss->mma_done);
      }
      wait_mma();
      if (et == 0 && ok && c + 2 < nchunks) {     // K of stage s is consumed
        load_k(c + 2);
        loaded_k = c + 3;
      }
      // (d) S -> bf16 copy for the next chunk's products;  O = scale * D_Q -> registers
      float oo[32];
      {
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          float v[32];
          if (ok) tmem_ld32_sync(s_addr + h2 * 32, v);
          else {
#pragma unroll
            for (int u = 0; u < 32; ++u) v[u] = 0.f;
          }
          write_sb(v, h2);
        }
        if (ok) {
          tmem_ld32_sync(tmem + lane_base + kColPair + hh * 32, oo);
          float z[32];
#pragma unroll
          for (int u = 0; u < 32; ++u) z[u] = 0.f;
          tmem_st32_sync(tmem + lane_base + kColPair + hh * 32, z);   // D_Q of chunk c + 1 starts at 0
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) oo[u] = 0.f;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarEpi, kNumEpi);
      // O staging (row j = token, 256 B per row) then coalesced 16-byte stores; the
      // prescale of S for the next chunk overlaps its first product
      write_o = it.write_o && t0 >= it.s && p.o != nullptr;
      if (write_o) {
        // token rows, two 64-column halves, 128B-swizzled (the layout of the TMA tile store)
        uint8_t* stg = sm + kOffDt + (r >> 6) * 8192 + (r & 7) * 2;
        const int rc = (r & 63) >> 3;
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int i = hh * 32 + jj;
          *reinterpret_cast<__nv_bfloat16*>(stg + i * 128 + ((rc ^ (i & 7)) << 4)) = __float2bfloat16_rn(p.scale * oo[jj]);
        }
      }
      // a full chunk's O leaves through two TMA tile stores as soon as the staging is fenced
      // (inside store_w when a chunk follows); their reads are waited for before this
      // iteration's last barrier, since the next chunk's step (b) rewrites the staging
      o_tma = write_o && nv == kChunk;
      }
      const bool next = c + 1 < nchunks;
      auto store_o = [&]() {
        tma_store_3d(&tm_o, sbase + kOffDt, 0, it.j, it.b * p.T + t0);
        tma_store_3d(&tm_o, sbase + kOffDt + 8192u, 64, it.j, it.b * p.T + t0);
        bulk_commit();
      };
      if (next) {
        // Q~ = diag(exp(gam)) Q of the next chunk (times rq under the normalisation), in place, while
        // the chain would otherwise wait for the prep: its Gram product has read Q and its decays are
        // written (dec_ready); store_w's fence and barrier order it before the first product
        const int s1 = (c + 1) & 1;
        ok = ok && mbar_wait(&ss->dec_ready[s1], ((c + 1) >> 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) scale_rows_tile_part(sm + s1 * kStageBytes + kOffQ, kHalf, kNorm ? ss->cs.egq[s1] : ss->cs.eg[s1], 1.f,
                                     et, kNumEpi);
        ok = ok && mbar_wait(&ss->prep_full[s1], ((c + 1) >> 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        // A2 = A diag(beta), B2 = A diag(beta exp(gam)) in bf16 from the prep's fp32 A, then
        // U^T = V^T A2^T into the Delta accumulator (chunk c's Delta was read in step (b)) and
        // W = B2 K into the chunk's G/W buffer (the previous U, W products completed before
        // store_w(c), so A2 and B2 are free)
        prep_store_a_f32<kNorm>(ec, s1, reinterpret_cast<const float*>(sm + kOffAst), sbase + kOffA2, sbase + kOffB2);
        fence_proxy_async_smem();
        named_bar_sync(kBarEpi, kNumEpi);
        if (et == 0 && ok) {
          mbar_arrive(&ss->a_free);
          tc_fence_after();
          const uint32_t st1 = sbase + s1 * kStageBytes;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            if (!it.zero_v)
              umma_f16(tmem + kColDd, sdesc_sw128(st1 + kOffV + ks * 2048, kHalf, 1024),
                       sdesc_sw128(sbase + kOffA2 + ks * 32, 16, 1024), kIdU, ks > 0);
            umma_f16(tmem + kColGW + 128u * s1, sdesc_sw128(sbase + kOffB2 + ks * 32, 16, 1024),
                     sdesc_sw128(st1 + ks * 2048, kHalf, 1024), kIdW, ks > 0);
          }
          umma_commit(&ss->wdone);
        }
        if (it.zero_v && ok) {                    // V = 0: the Delta accumulator starts from zero
          tc_fence_after();
          float z[32];
#pragma unroll
          for (int u = 0; u < 32; ++u) z[u] = 0.f;
          tmem_st32_sync(tmem + lane_base + kColDd + 32 * hh, z);
        }
        store_w(c + 1);
        if (et == 0 && ok && o_tma) store_o();
        if (et == 0 && ok) issue_a(c + 1);
      }
      if (next && ok) prescale((c + 1) & 1);
      if (c < 0) {
        tc_fence_before();
        continue;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarEpi, kNumEpi);
      if (write_o && ok) {
        if (o_tma) {
          if (et == 0 && !next) store_o();          // the last chunk
        } else {                                    // rows past the end belong to other data
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.o);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int idx = et + k4 * kNumEpi;
            const int j = idx >> 4, ch = idx & 15;
            if (j < nv) {
              const uint4 val =
                  *reinterpret_cast<const uint4*>(sm + kOffDt + (ch >> 3) * 8192 + j * 128 + (((ch & 7) ^ (j & 7)) << 4));
              *reinterpret_cast<uint4*>(o + ((size_t)(it.b * p.T + t0 + j) * p.Hv + it.j) * 128 + ch * 8) = val;
            }
          }
        }
      }
      if (et == 0) bulk_wait_read();                // the next chunk's step (b) rewrites the O staging
      named_bar_sync(kBarEpi, kNumEpi);
    }
    if (ok && it.fin != nullptr) {
      tc_fence_after();
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        float v[32];
        tmem_ld32_sync(s_addr + h2 * 32, v);
#pragma unroll
        for (int d = 0; d < 32; ++d) it.fin[(size_t)(hh * 64 + h2 * 32 + d) * 128 + r] = v[d];
      }
    }
    if (et == 0) bulk_wait_all();
    if (et == 0 && !ok) {
      // aborted: do not leave the CTA with copies in flight (bounded wait, flag ignored)
      volatile int never = 0;
      for (int c = (loaded_k >= 2 ? loaded_k - 2 : 0); c < loaded_k; ++c)
        mbar_wait(&ss->full_k[c & 1], (c >> 1) & 1, &never);
      for (int c = (loaded_qv >= 2 ? loaded_qv - 2 : 0); c < loaded_qv; ++c)
        mbar_wait(&ss->full_qv[c & 1], (c >> 1) & 1, &never);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) report_error(p, kDevTimeout);
}

// ---------------------------------------------------------------- host side
namespace {

}  // namespace

cudaError_t launch_fwd_tc(const FwdParams& p, const TcPlan& plan, int num_items, cudaStream_t st,
                          const char** what) {
  if (num_items <= 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  const long long rows = (long long)p.B * p.T;
  *what = "tensor map encode";
  if (!make_tile_map(&mq, p.q, p.Hqk, rows) || !make_tile_map(&mk, p.k, p.Hqk, rows) ||
      !make_tile_map(&mv, p.v, p.Hv, rows))
    return cudaErrorInvalidValue;
  CUtensorMap mo = mq;                       // o, same tiling as v (unused without o)
  if (p.o != nullptr && !make_tile_map(&mo, p.o, p.Hv, rows)) return cudaErrorInvalidValue;
  // chunk start states (bf16 [slots * Hv * 128 rows][128]): 128-row x 64-column boxes
  CUtensorMap ms = mq;                       // unused unless states are stored
  if (p.states != nullptr) {
    const long long nch = (p.T + kChunk - 1) / kChunk;
    const long long slots = p.cu != nullptr ? nch + p.N : (long long)p.N * nch;
    if (!make_tile_map(&ms, p.states, 1, slots * p.Hv * 128, 128)) return cudaErrorInvalidValue;
  }
  *what = "shared memory attribute";
  auto kernel = p.qk_l2norm ? gdn_fwd_tc_kernel<true> : gdn_fwd_tc_kernel<false>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (err != cudaSuccess) return err;
  *what = "tensor-core forward launch";
  trace_pre(kKernFwdTc, st);
  kernel<<<num_items, kThreads, kSmemBytes, st>>>(mq, mk, mv, ms, mo, p, plan);
  err = cudaGetLastError();
  trace_post(st);
  return err;
}

}  // namespace gdn
