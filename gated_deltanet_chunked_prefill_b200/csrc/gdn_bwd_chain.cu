// Backward, part 1 of 2 (tensor cores): the reverse chain of the state gradient.
//
// With S (dv x dk) the state at a chunk's start, the chunk maps it to
//   S' = exp(gam_n) S + Delta^T diag(exp(gam_n - gam)) K,
//   Delta^T = (V^T - S K^T diag(exp(gam))) (A diag(beta))^T,  O^T = scale (S Q~^T + Delta^T P^T)
// (the forward's WY/UT chunk form, Q~ = diag(exp(gam)) Q). Its adjoint carries the state
// gradient dS' at the chunk's end back to the chunk's start:
//   dDelta^T = dS' K^T diag(exp(gam_n - gam)) + dO^T (scale P)
//   dY^T     = dDelta^T (A diag(beta))
//   dS       = exp(gam_n) dS' + dO^T (scale diag(exp(gam)) Q) - dY^T diag(exp(gam)) K
// which needs neither S nor V. One CTA runs one (sequence, v-head) unit, or one segment
// of it, from the last chunk to the first, and stores the bf16 dS' of every chunk (the
// gradient at the chunk's end) for the gradient kernel; the first segment ends with dh0.
// The chain's three dependent products per chunk and the state-independent prep mirror
// the forward kernel ("FlashQLA resource", section 3: fused warp-specialised kernels;
// section 5: backward with intra-card sequence parallelism).
//
// Parameter mapping (FwdParams reused): v = dO [B,T,Hv,dv]; h0 = dhT (nullable);
// hT = dh0 (nullable); states = per-chunk dS' (bf16, dv x dk, required); o unused.
// Context parallelism mirrors the forward in reverse: a segment that ends inside the
// sequence starts from a zero gradient at the end of a window of later chunks whose
// decay bound is below 2^-64 (the transition's adjoint has the same norm), else at the
// sequence end from dhT.
#include <cudaTypedefs.h>

#include "gdn_chunk_prep.cuh"
#include "gdn_common.cuh"
#include "gdn_tc.cuh"
#include "tc_ptx.cuh"

namespace gdn {
using namespace tc;

namespace {

constexpr int kThreads = 512;
constexpr int kEpiWarp0 = 8;
constexpr int kNumPrep = 256, kNumEpi = 256;
constexpr int kBarPrep = 1, kBarEpi = 2;

constexpr uint32_t kStageBytes = 48u * 1024u;   // [K0 Q0 K1 Q1] + [dO0 dO1]
constexpr uint32_t kOffDO = 32u * 1024u;        // within a stage
constexpr uint32_t kOffA2 = 96u * 1024u;        // 2 x 8KB
constexpr uint32_t kOffP = 112u * 1024u;        // 2 x 8KB  P (from the forward pass)
constexpr uint32_t kOffSb = 128u * 1024u;       // 32KB  dS in bf16
constexpr uint32_t kOffDD = 160u * 1024u;       // 16KB  dDelta^T, bf16 [r][j]
constexpr uint32_t kOffDY = 176u * 1024u;       // 16KB  -dY^T diag(exp(gam)), bf16 [r][j]
constexpr uint32_t kOffLf = 192u * 1024u;
constexpr uint32_t kOffSmall = kOffLf + 64u * kLd * 4u;

struct Small {
  ChunkScalars cs;
  float wsum[16];
  uint64_t full[2], prep_full[2], gdone, mma_done;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr uint32_t kSmemBytes = kOffSmall + sizeof(Small);
static_assert(kSmemBytes <= 232448, "dynamic shared memory above the 227 KB a block can opt into");

constexpr uint32_t kColG = 0;     // 64: unused (the Gram product of the prep runs in the forward)
constexpr uint32_t kColDa = 64;   // 64: dS' K^T
constexpr uint32_t kColDb = 128;  // 64: dO^T P (scale applied when combined)
constexpr uint32_t kColDY = 192;  // 64: dDelta^T A2
constexpr uint32_t kColS = 256;   // 128: dS (dv x dk) fp32, updated in place
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kId64 = idesc_bf16(128, 64, false, false);
constexpr uint32_t kId64mm = idesc_bf16(128, 64, true, true);      // A and B MN-major
constexpr uint32_t kId64km = idesc_bf16(128, 64, false, true);     // B MN-major
constexpr uint32_t kId128mm = idesc_bf16(128, 128, true, true);
constexpr uint32_t kId128km = idesc_bf16(128, 128, false, true);

}  // namespace

// kNorm: q and k rows are L2-normalised in the kernel (their inverse norms folded into the
// per-token factors: egd and egk carry rk, the scaled Q tile carries rq).
template <bool kNorm>
__global__ void __launch_bounds__(kThreads, 1)
gdn_bwd_chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_s,
                     const FwdParams p, const TcPlan plan) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  Small* ss = reinterpret_cast<Small*>(sm + kOffSmall);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if ((smem_u32(sm) & 1023u) != 0) {
    if (threadIdx.x == 0) report_error(p, kDevMisaligned);
    return;
  }
  // Decode the work item. Exact stitch (phases 1 and 3): the reverse item gives the end gradient
  // (init) and where the start gradient goes (fin). Otherwise decode with h0/hT hidden (dhT / dh0
  // belong to the other ends here) and take them below.
  const bool exact = plan.kind == kPlanCpP1 || plan.kind == kPlanCpP3;
  FwdParams pd = p;
  pd.h0 = nullptr;
  pd.hT = nullptr;
  if (plan.seg_ws != nullptr && plan.kind == kPlanCpP1) {
    // exact fallback, phase 1: item = (pi * 2 + role) * Hv + j. When the window after the
    // predecessor's end closes (the probe's record, read first) no map is needed: leave at once.
    const int j = blockIdx.x % p.Hv, pi = blockIdx.x / (2 * p.Hv);
    if (pi >= 1 && plan.seg_ws[(size_t)(pi - 1) * p.Hv + j] >= 0) return;
  }
  WorkItem it;
  if (!get_work_item(exact ? p : pd, plan, blockIdx.x, it, exact)) return;
  const __nv_bfloat16* beta = static_cast<const __nv_bfloat16*>(p.beta);
  const bool is_first = it.s == it.seq_s, is_last = it.e == it.seq_e;
  const bool zero_do = exact && it.zero_v;             // transition role: dO = 0
  const bool store_ds = plan.kind != kPlanCpP1;        // phase 1 only maps the segment

  // End (exclusive) of the processed range, decided before any setup. Gate-driven plan: a segment
  // that ends inside the sequence starts from a zero gradient at the end of a window of later
  // chunks whose decay bound is below 2^-64, else at the sequence end from dhT. With the exact
  // stitch as fallback (plan.seg_ws, every segment's window after its end recorded by the probe
  // kernel), the mirror of the forward: in phase 1, when the window after the predecessor's end (this
  // segment's start) closes, the predecessor needs no end gradient and the CTA leaves; otherwise the
  // segment's map is computed, or its start gradient straight from its own window (role 0). Phase 3
  // starts from the window or from the stitched gradient.
  int we = it.e;
  if (it.gate) {
    if (!is_last) {
      const int w = gate_window_end(p, it, it.e, ss->wsum);
      we = w >= 0 ? w : it.seq_e;
    }
  } else if (plan.seg_ws != nullptr && plan.kind == kPlanCpP1) {
    if (plan.seg_ws[(size_t)(it.pi - 1) * p.Hv + it.j] >= 0) return;
    if (it.seg + 1 < it.segs_used) {
      const int w0 = plan.seg_ws[(size_t)it.pi * p.Hv + it.j];
      if (w0 >= 0) {
        if (it.role == 1) return;
        we = w0;
      }
    }
  } else if (plan.seg_ws != nullptr && plan.kind == kPlanCpP3 && it.seg + 1 < it.segs_used) {
    const int w = plan.seg_ws[(size_t)it.pi * p.Hv + it.j];
    if (w >= 0) we = w;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ss->full[s], 1);
      mbar_init(&ss->prep_full[s], 1);
    }
    mbar_init(&ss->gdone, 1);
    mbar_init(&ss->mma_done, 1);
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
    prefetch_tmap(&tm_do);
  }
  if (zero_do) {                                      // both stages' dO tiles: 2 x 16 KB of zeros
    for (int idx = threadIdx.x; idx < 2 * 1024; idx += kThreads)
      *reinterpret_cast<uint4*>(sm + (idx >> 10) * kStageBytes + kOffDO + (idx & 1023) * 16) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int nchunks = (we - it.s + kChunk - 1) / kChunk;   // chunk c covers [s + 64c, min(s + 64c + 64, we))
  const bool from_seq_end = we == it.seq_e;
  int init_mode = kInitZero;
  const float* init_ptr = nullptr;
  float* dh0 = nullptr;                                    // destination of the start gradient
  if (exact) {
    if (we == it.e) {                                    // from the item's end gradient
      init_mode = it.init_mode;
      init_ptr = it.init;
    } else if (from_seq_end && p.h0) {                   // from a window that reaches the sequence end
      init_mode = kInitPtr;
      init_ptr = p.h0 + ((size_t)it.n * p.Hv + it.j) * (size_t)(128 * 128);
    }
    dh0 = it.fin;
  } else {
    if (from_seq_end && p.h0) {
      init_mode = kInitPtr;
      init_ptr = p.h0 + ((size_t)it.n * p.Hv + it.j) * (size_t)(128 * 128);
    }
    if (is_first && p.hT) dh0 = p.hT + ((size_t)it.n * p.Hv + it.j) * (size_t)(128 * 128);
  }

  const uint32_t tmem = ss->tmem_base;
  volatile int* abort_flag = &ss->abort_flag;
  const uint32_t sbase = smem_u32(sm);

  // processing step k handles chunk c = nchunks - 1 - k, in stage k % 2
  auto chunk_of = [&](int k) { return nchunks - 1 - k; };
  auto load_step = [&](int k) {
    const int s = k & 1;
    const int row = it.b * p.T + it.s + chunk_of(k) * kChunk;
    uint8_t* st = sm + s * kStageBytes;
    mbar_arrive_expect_tx(&ss->full[s], zero_do ? kOffDO : kStageBytes);
    tma_load_3d(st + 0, &tm_k, &ss->full[s], 0, it.hq, row);
    tma_load_3d(st + 8192, &tm_q, &ss->full[s], 0, it.hq, row);
    tma_load_3d(st + 16384, &tm_k, &ss->full[s], 64, it.hq, row);
    tma_load_3d(st + 24576, &tm_q, &ss->full[s], 64, it.hq, row);
    if (!zero_do) {                                   // dO = 0: its tiles stay zero (cleared at the start)
      tma_load_3d(st + kOffDO, &tm_do, &ss->full[s], 0, it.j, row);
      tma_load_3d(st + kOffDO + 8192, &tm_do, &ss->full[s], 64, it.j, row);
    }
  };

  if (warp < kEpiWarp0) {
    // ------------------------------------------------------------ prep (8 warps)
    const int pt = threadIdx.x;
    PrepCtx pc{sbase, reinterpret_cast<float*>(sm + kOffLf), &ss->cs, tmem, kColG, pt, warp, lane, kBarPrep};
    bool ok = true;
    // g, beta of chunk k (0 past the segment's end), loaded one chunk ahead
    auto load_gb = [&](int k, float& gv, float& bv) {
      gv = 0.f;
      bv = 0.f;
      if (k >= nchunks) return;
      const int t0 = it.s + chunk_of(k) * kChunk;
      if (pt < kChunk && pt < min(kChunk, we - t0)) {
        const size_t gi = (size_t)(it.b * p.T + t0 + pt) * p.Hv + it.j;
        gv = p.g[gi];
        bv = __bfloat162float(beta[gi]);
      }
    };
    float gv_next = 0.f, bv_next = 0.f;
    load_gb(0, gv_next, bv_next);
    for (int k = 0; k < nchunks; ++k) {
      const int s = k & 1;
      const int t0 = it.s + chunk_of(k) * kChunk;
      const int nv = min(kChunk, we - t0);
      uint8_t* st = sm + s * kStageBytes;
      // A = (I + L)^-1 of this chunk, as the forward pass computed it (same arithmetic)
      prep_fetch_a(pc, p.chunk_a + (chunk_slot(p, it.n, (t0 - it.seq_s) / kChunk) * p.Hv + it.j) *
                                       (size_t)(kChunk * kChunk));
      const float gv = gv_next, bv = bv_next;
      load_gb(k + 1, gv_next, bv_next);
      ok = ok && mbar_wait(&ss->full[s], (k >> 1) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      // P = lower_incl(Q K^T * E) of this chunk from the forward pass (bf16 operand tile); its
      // slot was last read by chunk k - 2's first product, complete once these tiles landed
      {
        const uint8_t* pg = p.chunk_p + (chunk_slot(p, it.n, (t0 - it.seq_s) / kChunk) * p.Hv + it.j) * (size_t)8192;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const int idx = pt + kNumPrep * m;
          tc::cp_async_16(sbase + kOffP + s * 8192u + idx * 16u, pg + idx * 16);
        }
        tc::cp_async_commit();
      }
      prep_store_gb(pc, s, gv, bv);
      if (nv < kChunk) {
        for (int idx = pt; idx < (kChunk - nv) * 48; idx += kNumPrep) {
          const int r = nv + idx / 48, rem = idx % 48, tile = rem / 8, ch = rem % 8;
          const uint32_t off = (tile < 4 ? tile * 8192u : kOffDO + (tile - 4) * 8192u) + r * 128u + ch * 16u;
          *reinterpret_cast<uint4*>(st + off) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      named_bar_sync(kBarPrep, kNumPrep);
      if (kNorm) row_inv_norms(st, st + 16384, st + 8192, st + 24576, ss->cs.rk[s], ss->cs.rq[s], pt);
      prep_scan(pc, s);
      named_bar_sync(kBarPrep, kNumPrep);
      prep_decays<kNorm>(pc, s, nv);
      named_bar_sync(kBarPrep, kNumPrep);
      // Q <- scale diag(exp(gam)) Q (times rq under the normalisation)
      scale_rows_tile_part(st + 8192, 16384, kNorm ? ss->cs.egq[s] : ss->cs.eg[s], p.scale, pt, kNumPrep);
      tc::cp_async_wait_all();
      named_bar_sync(kBarPrep, kNumPrep);
      prep_write_a_rows(pc, s, sbase + kOffA2 + s * 8192u, 0);                       // A diag(beta)
      fence_proxy_async_smem();
      named_bar_sync(kBarPrep, kNumPrep);
      if (pt == 0 && ok) mbar_arrive(&ss->prep_full[s]);
    }
  } else {
    // ------------------------------------------------------------ epilogue: the gradient chain
    const int et = threadIdx.x - kEpiWarp0 * 32;
    const int ew = et >> 5;
    const int qd = ew & 3, hh = ew >> 2;
    const int r = 32 * qd + lane;
    const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
    const uint32_t s_addr = tmem + lane_base + kColS + hh * 64;
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
    // dS at the end of the processed range: dhT^T (sequence end) or 0
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
    fence_proxy_async_smem();
    tc_fence_before();
    named_bar_sync(kBarEpi, kNumEpi);
    uint32_t mph = 0;
    // (1) Da = dS' K^T ;  Db = dO^T P
    auto issue_1 = [&](int k) {
      tc_fence_after();
      const uint32_t a0 = sbase + kOffSb, st = sbase + (k & 1) * kStageBytes;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t off = (ks >> 2) * 16384u + (ks & 3) * 32u;
        umma_f16(tmem + kColDa, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(st + off, 16, 1024), kId64, ks > 0);
      }
      const uint32_t dob = st + kOffDO, pb = sbase + kOffP + (k & 1) * 8192u;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        umma_f16(tmem + kColDb, sdesc_sw128(dob + ks * 2048, 8192, 1024), sdesc_sw128(pb + ks * 2048, 8192, 1024),
                 kId64mm, ks > 0);
      umma_commit(&ss->mma_done);
    };
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
    int loaded = 0;
    if (et == 0) {
      for (; loaded < 2 && loaded < nchunks; ++loaded) load_step(loaded);
    }
    if (nchunks > 0) {
      ok = mbar_wait(&ss->prep_full[0], 0, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (et == 0 && ok) issue_1(0);
      if (ok) prescale(0);
      tc_fence_before();
    }
    auto wait_mma = [&]() {
      ok = ok && mbar_wait(&ss->mma_done, mph, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      mph ^= 1;
      tc_fence_after();
    };
    for (int k = 0; k < nchunks; ++k) {
      const int s = k & 1;
      const int c = chunk_of(k);
      const int t0 = it.s + c * kChunk;
      wait_mma();
      if (et == 0 && t0 < it.e && ok && store_ds) {
        // dS' of this chunk (its end gradient) for the gradient kernel: two TMA tile stores
        // from the swizzled bf16 copy, waited for (reads) before the copy is rewritten
        const int srow = (int)((chunk_slot(p, it.n, (t0 - it.seq_s) / kChunk) * p.Hv + it.j) * 128);
        tma_store_3d(&tm_s, sbase + kOffSb, 0, 0, srow);
        tma_store_3d(&tm_s, sbase + kOffSb + 16384u, 64, 0, srow);
        bulk_commit();
      }
      // dDelta^T = Da diag(exp(gam_n - gam)) + Db  -> bf16
      {
        float da[32], db[32];
        if (ok) {
          tmem_ld32_sync(tmem + lane_base + kColDa + hh * 32, da);
          tmem_ld32_sync(tmem + lane_base + kColDb + hh * 32, db);
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) da[u] = db[u] = 0.f;
        }
        const float* egd = ss->cs.egd[s];
        uint32_t w[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int j0 = hh * 32 + 2 * u;
          w[u] = pack_bf16(fmaf(da[2 * u], egd[j0], p.scale * db[2 * u]),
                           fmaf(da[2 * u + 1], egd[j0 + 1], p.scale * db[2 * u + 1]));
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          st_shared_v4(sbase + kOffDD + sw128(r, hh * 4 + c4), w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarEpi, kNumEpi);
      // (2) dY^T = dDelta^T (A diag(beta))
      if (et == 0 && ok) {
        tc_fence_after();
        const uint32_t a0 = sbase + kOffDD, b0 = sbase + kOffA2 + s * 8192u;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_f16(tmem + kColDY, sdesc_sw128(a0 + ks * 32, 16, 1024), sdesc_sw128(b0 + ks * 2048, 8192, 1024),
                   kId64km, ks > 0);
        umma_commit(&ss->mma_done);
      }
      wait_mma();
      // -dY^T diag(exp(gam)) -> bf16 (times rk under the normalisation: it multiplies the raw K)
      {
        float dy[32];
        if (ok) tmem_ld32_sync(tmem + lane_base + kColDY + hh * 32, dy);
        else {
#pragma unroll
          for (int u = 0; u < 32; ++u) dy[u] = 0.f;
        }
        const float* eg = kNorm ? ss->cs.egk[s] : ss->cs.eg[s];
        uint32_t w[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int j0 = hh * 32 + 2 * u;
          w[u] = pack_bf16(-dy[2 * u] * eg[j0], -dy[2 * u + 1] * eg[j0 + 1]);
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          st_shared_v4(sbase + kOffDY + sw128(r, hh * 4 + c4), w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
      }
      if (et == 0) bulk_wait_read();                // the dS' copy is rewritten after this barrier
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarEpi, kNumEpi);
      // (3) dS += dO^T (scale diag(exp(gam)) Q) + (-dY^T diag(exp(gam))) K   (dS pre-scaled by exp(gam_n))
      if (et == 0 && ok) {
        tc_fence_after();
        const uint32_t st = sbase + s * kStageBytes;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_f16(tmem + kColS, sdesc_sw128(st + kOffDO + ks * 2048, 8192, 1024),
                   sdesc_sw128(st + 8192 + ks * 2048, 16384, 1024), kId128mm, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_f16(tmem + kColS, sdesc_sw128(sbase + kOffDY + ks * 32, 16, 1024),
                   sdesc_sw128(st + ks * 2048, 16384, 1024), kId128km, 1);
        umma_commit(&ss->mma_done);
      }
      wait_mma();
      // dS -> bf16 for the next (earlier) chunk
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
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(kBarEpi, kNumEpi);
      const bool next = k + 1 < nchunks;
      if (et == 0 && ok && k + 2 < nchunks) {
        load_step(k + 2);
        loaded = k + 3;
      }
      if (next) {
        ok = ok && mbar_wait(&ss->prep_full[(k + 1) & 1], ((k + 1) >> 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (et == 0 && ok) issue_1(k + 1);
        if (ok) prescale((k + 1) & 1);
      }
      tc_fence_before();
      named_bar_sync(kBarEpi, kNumEpi);
    }
    if (ok && dh0 != nullptr) {
      tc_fence_after();
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        float v[32];
        tmem_ld32_sync(s_addr + h2 * 32, v);
#pragma unroll
        for (int d = 0; d < 32; ++d) dh0[(size_t)(hh * 64 + h2 * 32 + d) * 128 + r] = v[d];
      }
    }
    if (et == 0) bulk_wait_all();
    if (et == 0 && !ok) {
      for (int k = (loaded >= 2 ? loaded - 2 : 0); k < loaded; ++k) {
        volatile int never = 0;
        mbar_wait(&ss->full[k & 1], (k >> 1) & 1, &never);
      }
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

cudaError_t launch_bwd_chain(const FwdParams& p, const TcPlan& plan, int num_items, cudaStream_t st,
                             const char** what) {
  if (num_items <= 0) return cudaSuccess;
  CUtensorMap mq, mk, mdo;
  const long long rows = (long long)p.B * p.T;
  *what = "tensor map encode";
  if (!make_tile_map(&mq, p.q, p.Hqk, rows) || !make_tile_map(&mk, p.k, p.Hqk, rows) ||
      !make_tile_map(&mdo, p.v, p.Hv, rows))
    return cudaErrorInvalidValue;
  // per-chunk dS' (bf16 [slots * Hv * 128 rows][128]): 128-row x 64-column boxes
  CUtensorMap ms;
  {
    const long long nch = (p.T + kChunk - 1) / kChunk;
    const long long slots = p.cu != nullptr ? nch + p.N : (long long)p.N * nch;
    if (!make_tile_map(&ms, p.states, 1, slots * p.Hv * 128, 128)) return cudaErrorInvalidValue;
  }
  *what = "shared memory attribute";
  auto kernel = p.qk_l2norm ? gdn_bwd_chain_kernel<true> : gdn_bwd_chain_kernel<false>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (err != cudaSuccess) return err;
  *what = "backward chain launch";
  trace_pre(kKernBwdChain, st);
  kernel<<<num_items, kThreads, kSmemBytes, st>>>(mq, mk, mdo, ms, p, plan);
  err = cudaGetLastError();
  trace_post(st);
  return err;
}

}  // namespace gdn
