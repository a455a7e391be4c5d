// Backward, part 2 of 2 (tensor cores): the gradients of one 64-token chunk of one
// (sequence, v-head), given the chunk's start state S and the state gradient dS' at its
// end (both bf16, dv x dk, written by the state pass and the reverse chain). Chunks are
// independent here, so the grid covers every (chunk, v-head) at once.
//
// Forward of the chunk (S-form, gam = inclusive cumsum of g, E_ij = exp(gam_i - gam_j)):
//   L = strict_lower(diag(beta) KK^T * E), A = (I + L)^-1, A2 = A diag(beta)
//   Y^T = V^T - S K^T diag(e^gam),  Delta^T = Y^T A2^T
//   O^T = scale (S Q^T diag(e^gam) + Delta^T P^T),  P = lower_incl(QK^T * E)
//   S'  = e^gam_n S + Delta^T diag(e^(gam_n - gam)) K
// Adjoint (dO, dS' given; dP = scale dO Delta^T, dPm = dP * E * lower_incl):
//   dDelta^T = dS' K^T diag(e^(gam_n - gam)) + dO^T (scale P);   dY^T = dDelta^T A2
//   dV = dY;  dA2 = dDelta Y^T;  dbeta_j += sum_i dA2_ij A_ij;  dA = dA2 diag(beta)
//   dL = -A^T dA A^T (strictly lower);  dG = dL * beta_i E (i > j);  dbeta_i += sum_j dL_ij KK_ij E_ij
//   dQ = scale diag(e^gam) dO S + dPm K
//   dK = dPm^T Q + (dG + dG^T) K - diag(e^gam) dY S + diag(e^(gam_n - gam)) Delta dS'
//   dgam_i += scale e^gam_i sum_r dO_ir (S Q^T)_ri - e^gam_i sum_r dY_ir (S K^T)_ri
//            + sum_j (F_ij - F_ji),  F = dP * P + dL * L
//   dgam_j -= s_j,  dgam_{n} += sum_j s_j + e^gam_n <S, dS'>,  s_j = e^(gam_n - gam_j) sum_r Delta_jr (dS' K^T)_rj
//   dg = reverse cumsum of dgam within the chunk.
// (The oracle's token adjoint is the reference semantics; this is its chunked form.)
//
// All products are tcgen05 MMAs with 128 TMEM lanes: a product with 64 meaningful rows reads
// 64 further rows of whatever follows in shared memory and ignores those lanes.
#include <cudaTypedefs.h>

#include <algorithm>

#include "gdn_chunk_prep.cuh"
#include "gdn_common.cuh"
#include "gdn_tc.cuh"
#include "tc_ptx.cuh"

namespace gdn {
using namespace tc;

namespace {

constexpr int kThreads = 256;
constexpr int kBar = 1;
constexpr int kLateIssuer = 64;   // lane 0 of warp 2 (TMEM lanes 64..95: no rows in the dL phase)

// shared memory (bytes from the 1024-aligned base)
constexpr uint32_t kOffKQ = 0;            // [K0 Q0 K1 Q1]
constexpr uint32_t kOffVDO = 32u * 1024;  // [V0 dO0 V1 dO1]; V0/V1 become dD0/dD1 (dDelta, token-major)
constexpr uint32_t kOffS = 64u * 1024;    // S  [r][d] bf16, two 16KB column halves
constexpr uint32_t kOffDS = 96u * 1024;   // dS'
constexpr uint32_t kOffYt = 128u * 1024;  // Y^T [r][j]; then -e^gam dY^T
constexpr uint32_t kOffDt = 144u * 1024;  // Delta^T [r][j]; then e^(gam_n - gam) Delta^T
constexpr uint32_t kOffA2 = 160u * 1024;  // A diag(beta)
constexpr uint32_t kOffP = 168u * 1024;   // P (from the forward pass); then dPm
constexpr uint32_t kOffA = 176u * 1024;   // A; then dG + dG^T
constexpr uint32_t kOffDA = 184u * 1024;  // dA; then X = dA A^T
constexpr uint32_t kOffLf = 192u * 1024;  // A (fp32, the forward's swizzled 64 x 64 layout); then dG (64 x kLd)
constexpr uint32_t kOffSmall = kOffLf + 64u * kLd * 4u;

// Per-token partial sums, one slot per producer so that every slot entry is written exactly
// once and the final sums run in a fixed order (bit-reproducible results).
enum : int { kSlotTok = 0, kSlotFP = 4, kSlotFPRow = 6, kSlotFL = 8, kSlotFLRow = 10, kNumGamSlots = 12 };
enum : int { kSlotBetaA = 0, kSlotBetaL = 2, kNumBetaSlots = 4 };

struct Small {
  ChunkScalars cs;
  float dgam[kNumGamSlots][64];
  float dbeta[kNumBetaSlots][64];
  float dgn[16];
  float pdot[2][2][64];   // q/k normalisation: per (dq | dk, column half, row) partial dot products
  uint64_t tma_bar, mma_bar, gram_bar;   // gram_bar: the Gram product's own commit (its
                                         // completion is implied by the next mma_bar phase)
  uint32_t tmem_base;
  int abort_flag;
  int next[10];           // this CTA's next item, its position (n, c, j, b, s0, e0) and its tile rows
                          // (row, hq, srow), from warp 3
};
constexpr uint32_t kSmemBytes = kOffSmall + sizeof(Small);
static_assert(kSmemBytes <= 232448, "dynamic shared memory above the 227 KB a block can opt into");

// TMEM columns
constexpr uint32_t kColG = 0;     // [K;Q] K^T (64)
constexpr uint32_t kColY = 64;    // S K^T (64), with S Q^T next to it: one S [K;Q]^T product
constexpr uint32_t kColSQ = 128;  // S Q^T (64)
constexpr uint32_t kColDt = 192;  // Delta^T (64)
constexpr uint32_t kColD = 128;   // [dDelta;dO][Y^T|Delta^T] (128): dA2 | dP, after S Q^T and Delta^T are read
constexpr uint32_t kColDa = 256;  // dS' K^T (64); later X (64)
constexpr uint32_t kColDb = 320;  // dO^T P (64); later dY^T (64); later dL (64)
constexpr uint32_t kColQ = 384;   // dQ (128)
constexpr uint32_t kColK = 128;   // dK (128), after dA2/dP are consumed
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ uint64_t kdesc(uint32_t a) { return sdesc_sw128(a, 16, 1024); }
__device__ __forceinline__ uint64_t mdesc(uint32_t a, uint32_t lbo) { return sdesc_sw128(a, lbo, 1024); }

// 32 values per lane -> lane l gets the sum over the warp's 32 lanes of value l.
__device__ __forceinline__ float warp_transpose_sum(float* v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = upper ? v[i] : v[i + w];
      const float recv = __shfl_xor_sync(0xffffffffu, send, w);
      v[i] = (upper ? v[i + w] : v[i]) + recv;
    }
  }
  return v[0];
}

}  // namespace

// kNorm: q and k rows are L2-normalised in the kernel. The products run on the raw tiles with the
// inverse row norms rk, rq folded into per-token factors: the dQ accumulator holds rq * dQn and the
// dK accumulator rk * dKn (dQn, dKn: gradients w.r.t. the normalised rows), and the raw-row
// gradients are x - xn (xn . x) of those, with xn the normalised row.
template <bool kNorm>
__global__ void __launch_bounds__(kThreads, 1)
gdn_bwd_grad_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_ds,
                    const __grid_constant__ CUtensorMap tm_dv, const __grid_constant__ CUtensorMap tm_dq,
                    const __grid_constant__ CUtensorMap tm_dk, const FwdParams p, const BwdOut out,
                    const int num_items) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  Small* ss = reinterpret_cast<Small*>(sm + kOffSmall);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hh = warp >> 2;
  if ((smem_u32(sm) & 1023u) != 0) {
    if (tid == 0) report_error(p, kDevMisaligned);
    return;
  }
  if (tid == 0) {
    mbar_init(&ss->tma_bar, 1);
    mbar_init(&ss->mma_bar, 1);
    mbar_init(&ss->gram_bar, 1);
    ss->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ss->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ss->tmem_base;
  volatile int* abort_flag = &ss->abort_flag;
  const uint32_t sbase = smem_u32(sm);
  const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
  const int r = 32 * qd + lane;               // TMEM lane of this thread (M = 128 layouts)
  const __nv_bfloat16* beta = static_cast<const __nv_bfloat16*>(p.beta);
  // item = chunk_index * Hv + j -> (sequence n, chunk c of it, v-head j) and its token span
  struct Pos {
    int n, c, j, b, s0, e0;
  };
  auto decode = [&](int item, Pos& q) -> bool {
    q.j = item % p.Hv;
    const int gc = item / p.Hv;
    if (p.chunk_off) {                        // packed sequences: last n with chunk_off[n] <= gc
      int lo = 0, hi = p.N - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.chunk_off[mid] <= gc) lo = mid; else hi = mid - 1;
      }
      q.n = lo;
      q.c = gc - p.chunk_off[q.n];
    } else {
      const int nch = (p.T + kChunk - 1) / kChunk;
      q.n = gc / nch;
      q.c = gc % nch;
    }
    if (q.n >= p.N || q.c < 0) return false;
    if (!seq_span(p, q.n, q.b, q.s0, q.e0)) return false;
    return q.s0 + q.c * kChunk < q.e0;
  };
  // tiles of an item: K, Q (q/k head), V, dO (v-head) token rows; S, dS' state rows
  auto item_rows = [&](const Pos& q, int& row, int& hq, int& srow) {
    row = q.b * p.T + q.s0 + q.c * kChunk;
    hq = q.j / (p.Hv / p.Hqk);
    srow = (int)((chunk_slot(p, q.n, q.c) * p.Hv + q.j) * 128);
  };
  // decode() for one warp, scanning forward from sequence n0 (at most the item's own sequence: a
  // CTA's items visit nondecreasing sequences): 32 chunk offsets per round instead of a binary
  // search of dependent loads
  auto decode_warp = [&](int item, int n0, Pos& q) -> bool {
    q.j = item % p.Hv;
    const int gc = item / p.Hv;
    if (p.chunk_off) {                        // the last n with chunk_off[n] <= gc (offsets ascend)
      int base = n0;
      for (;;) {
        const int cand = base + 1 + lane;
        const unsigned m = __ballot_sync(0xffffffffu, cand < p.N && p.chunk_off[cand] <= gc);
        base += __popc(m);
        if (m != 0xffffffffu) break;
      }
      q.n = base;
      q.c = gc - p.chunk_off[base];
    } else {
      const int nch = (p.T + kChunk - 1) / kChunk;
      q.n = gc / nch;
      q.c = gc % nch;
    }
    if (q.n >= p.N || q.c < 0) return false;
    if (!seq_span(p, q.n, q.b, q.s0, q.e0)) return false;
    return q.s0 + q.c * kChunk < q.e0;
  };
  uint32_t mph = 0, tph = 0;
  // Persistent: this CTA takes the valid items among blockIdx.x, blockIdx.x + gridDim.x, ... (setup
  // and TMEM allocation once per CTA). From the second item on, warp 3 has found the item and formed
  // its gate scalars (in slot 1 of ChunkScalars, moved to slot 0 here) during the previous item.
  auto load_kq = [&](int hq, int row) {
    tma_load_3d(sm + kOffKQ + 0, &tm_k, &ss->tma_bar, 0, hq, row);
    tma_load_3d(sm + kOffKQ + 8192, &tm_q, &ss->tma_bar, 0, hq, row);
    tma_load_3d(sm + kOffKQ + 16384, &tm_k, &ss->tma_bar, 64, hq, row);
    tma_load_3d(sm + kOffKQ + 24576, &tm_q, &ss->tma_bar, 64, hq, row);
  };
  auto load_rest = [&](int j, int row, int srow) {
    tma_load_3d(sm + kOffVDO + 0, &tm_v, &ss->tma_bar, 0, j, row);
    tma_load_3d(sm + kOffVDO + 8192, &tm_do, &ss->tma_bar, 0, j, row);
    tma_load_3d(sm + kOffVDO + 16384, &tm_v, &ss->tma_bar, 64, j, row);
    tma_load_3d(sm + kOffVDO + 24576, &tm_do, &ss->tma_bar, 64, j, row);
    tma_load_3d(sm + kOffS, &tm_s, &ss->tma_bar, 0, 0, srow);
    tma_load_3d(sm + kOffS + 16384, &tm_s, &ss->tma_bar, 64, 0, srow);
    tma_load_3d(sm + kOffDS, &tm_ds, &ss->tma_bar, 0, 0, srow);
    tma_load_3d(sm + kOffDS + 16384, &tm_ds, &ss->tma_bar, 64, 0, srow);
  };
  // the forward's A (fp32, its swizzled 64 x 64 layout, kept as is) and P (the swizzled bf16 tile)
  auto load_ap = [&](int srow) {
    bulk_load(sbase + kOffLf, out.chunk_a + (size_t)srow / 128 * (kChunk * kChunk), kChunk * kChunk * 4u, &ss->tma_bar);
    bulk_load(sbase + kOffP, out.chunk_p + (size_t)srow / 128 * 8192, 8192u, &ss->tma_bar);
  };
  constexpr uint32_t kItemBytes = 128u * 1024u + kChunk * kChunk * 4u + 8192u;   // tiles, A, P
  bool prefetched = false;
  int item = blockIdx.x;
  Pos pos;
  while (item < num_items && !decode(item, pos)) item += gridDim.x;   // uniform over the CTA
  bool scal_ready = false;
  while (item < num_items) {
  if (scal_ready && tid < kChunk) {
    ChunkScalars& cs = ss->cs;
    cs.gam[0][tid] = cs.gam[1][tid];
    cs.egt[0][tid] = cs.egt[1][tid];
    cs.eg[0][tid] = cs.eg[1][tid];
    cs.egd[0][tid] = cs.egd[1][tid];
    cs.bet[0][tid] = cs.bet[1][tid];
    if (tid == 0) {
      cs.egn[0] = cs.egn[1];
      cs.nv[0] = cs.nv[1];
    }
  }
  if (tid == 0) bulk_wait_read();             // the previous item's output tiles have been read
  if (__syncthreads_or(*abort_flag)) break;
  const int j = pos.j, n = pos.n, c = pos.c, b = pos.b, e0 = pos.e0;
  int row, hq, srow;
  if (scal_ready) {
    row = ss->next[7];
    hq = ss->next[8];
    srow = ss->next[9];
  } else {
    item_rows(pos, row, hq, srow);
  }
  const int t0 = pos.s0 + c * kChunk;
  const int nv = min(kChunk, e0 - t0);
  (void)n;
  (void)b;
  if (!prefetched) {
    if (tid == 0) {
      mbar_arrive_expect_tx(&ss->tma_bar, kItemBytes);
      load_kq(hq, row);
      load_rest(j, row, srow);
      load_ap(srow);
    }
  } else if (kNorm && tid == 0) {
    load_kq(hq, row);
  }
  prefetched = false;
  PrepCtx pc{sbase, reinterpret_cast<float*>(sm + kOffLf), &ss->cs, tmem, kColG, tid, warp, lane, kBar};
  if (!scal_ready) {
    float gv = 0.f, bv = 0.f;
    if (tid < nv) {
      const size_t gi = (size_t)row * p.Hv + j + (size_t)tid * p.Hv;
      gv = p.g[gi];
      bv = __bfloat162float(beta[gi]);
    }
    prep_store_gb(pc, 0, gv, bv);
    // gam and the decay factors need only g: they run while the tiles are in flight
    __syncthreads();
    prep_scan(pc, 0);
    __syncthreads();
    prep_decays(pc, 0, nv);
  }
  bool ok = mbar_wait(&ss->tma_bar, tph, abort_flag);
  tph ^= 1;
  if (nv < kChunk) {                          // rows past the sequence end: zero
    ok = __syncthreads_and(ok);
    for (int idx = tid; idx < (kChunk - nv) * 64; idx += kThreads) {
      const int rr = nv + idx / 64, rem = idx % 64, tile = rem / 8, ch = rem % 8;
      *reinterpret_cast<uint4*>(sm + tile * 8192u + rr * 128u + ch * 16u) = make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async_smem();                   // zeroed rows are operands below
  ok = __syncthreads_and(ok);
  auto commit_wait = [&](int issuer = 0) {
    if (tid == issuer && ok) umma_commit(&ss->mma_bar);
    ok = ok && mbar_wait(&ss->mma_bar, mph, abort_flag);
    ok = __syncthreads_and(ok);
    mph ^= 1;
    tc_fence_after();
  };
  // ---- G = [K;Q] K^T and the products that need only the loaded tiles: S K^T, S Q^T,
  //      dS' K^T, dO^T P. G is first read after their commit, which also covers the Gram
  //      product issued before them.
  if (tid == 0 && ok) {
    issue_gram(tmem + kColG, sbase + kOffKQ, &ss->gram_bar);
    constexpr uint32_t id64 = idesc_bf16(128, 64, false, false);
    constexpr uint32_t id128 = idesc_bf16(128, 128, false, false);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t off = (ks >> 2) * 16384u + (ks & 3) * 32u;
      // B = [K;Q] (K then Q, 8KB apart): N = 128 gives S K^T and S Q^T in one series
      umma_f16(tmem + kColY, kdesc(sbase + kOffS + off), kdesc(sbase + kOffKQ + off), id128, ks > 0);
      umma_f16(tmem + kColDa, kdesc(sbase + kOffDS + off), kdesc(sbase + kOffKQ + off), id64, ks > 0);
    }
    // dO^T (scale P): A = dO MN-major (dv halves 16KB apart), B = scale P MN-major
    constexpr uint32_t idmm = idesc_bf16(128, 64, true, true);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      umma_f16(tmem + kColDb, mdesc(sbase + kOffVDO + 8192 + ks * 2048, 16384), mdesc(sbase + kOffP + ks * 2048, 8192),
               idmm, ks > 0);
  }
  // A (fp32 rows, from the forward pass) -> A diag(beta) and A in bf16
  // A (fp32) -> A diag(beta) and A in bf16 (128B-swizzled K-major rows); thread: row i, 16 columns
  {
    const int i = tid & 63, qq = tid >> 6;
    const float* af = reinterpret_cast<const float*>(sm + kOffLf);
    const float* bet = ss->cs.bet[0];
    float a[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 t = *reinterpret_cast<const float4*>(af + i * kChunk + a_chunk(i, qq * 4 + u) * 4);
      a[4 * u] = t.x; a[4 * u + 1] = t.y; a[4 * u + 2] = t.z; a[4 * u + 3] = t.w;
    }
    uint32_t w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) w[u] = pack_bf16(a[2 * u] * bet[qq * 16 + 2 * u], a[2 * u + 1] * bet[qq * 16 + 2 * u + 1]);
    st_shared_v4(sbase + kOffA2 + sw128(i, 2 * qq), w[0], w[1], w[2], w[3]);
    st_shared_v4(sbase + kOffA2 + sw128(i, 2 * qq + 1), w[4], w[5], w[6], w[7]);
#pragma unroll
    for (int u = 0; u < 8; ++u) w[u] = pack_bf16(a[2 * u], a[2 * u + 1]);
    st_shared_v4(sbase + kOffA + sw128(i, 2 * qq), w[0], w[1], w[2], w[3]);
    st_shared_v4(sbase + kOffA + sw128(i, 2 * qq + 1), w[4], w[5], w[6], w[7]);
  }
  if (kNorm) {
    // inverse row norms of K and Q, folded into the decay factors (egd, egk carry rk; egq rq)
    row_inv_norms(sm + kOffKQ, sm + kOffKQ + 16384, sm + kOffKQ + 8192, sm + kOffKQ + 24576, ss->cs.rk[0],
                  ss->cs.rq[0], tid);
    __syncthreads();
    if (tid < kChunk) {
      const float rk = ss->cs.rk[0][tid], e = ss->cs.eg[0][tid];
      ss->cs.egd[0][tid] *= rk;
      ss->cs.egk[0][tid] = e * rk;
      ss->cs.egq[0][tid] = e * ss->cs.rq[0][tid];
    }
  }
  fence_proxy_async_smem();
  commit_wait();
  const float* eg = ss->cs.eg[0];
  const float* egd = ss->cs.egd[0];
  const float* egk = kNorm ? ss->cs.egk[0] : eg;   // exp(gam), times rk under the normalisation
  const float* egq = kNorm ? ss->cs.egq[0] : eg;   // exp(gam), times rq under the normalisation
  // ---- Y^T = V^T - (S K^T) diag(e^gam);  dDelta = dS' K^T diag(e^(gam_n - gam)) + dO^T scale P
  float yv[32], ddv[32];
  {
    float sk[32], da[32], db[32];
    if (ok) {
      tmem_ld32_sync(tmem + lane_base + kColY + hh * 32, sk);
      tmem_ld32_sync(tmem + lane_base + kColDa + hh * 32, da);
      tmem_ld32_sync(tmem + lane_base + kColDb + hh * 32, db);
    } else {
#pragma unroll
      for (int u = 0; u < 32; ++u) sk[u] = da[u] = db[u] = 0.f;
    }
    const uint8_t* vt = sm + kOffVDO + (r >> 6) * 16384;
    const int rc = (r & 63) >> 3, rb = (r & 7) * 2;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int jj = hh * 32 + u;
      const float vv = bf16_at(vt + jj * 128 + ((rc ^ (jj & 7)) << 4) + rb);
      yv[u] = vv - egk[jj] * sk[u];
      ddv[u] = fmaf(da[u], egd[jj], p.scale * db[u]);      // P is unscaled
    }
  }
  __syncthreads();                            // every V read is done: dD may overwrite V
  {
    uint32_t w[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) w[u] = pack_bf16(yv[2 * u], yv[2 * u + 1]);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
      st_shared_v4(sbase + kOffYt + sw128(r, hh * 4 + c4), w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
    // dDelta token-major [i][r] in the V slots (dv half r / 64)
    uint8_t* dd = sm + kOffVDO + (r >> 6) * 16384;
    const int rc = (r & 63) >> 3, rb = (r & 7) * 2;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int ii = hh * 32 + u;
      *reinterpret_cast<__nv_bfloat16*>(dd + ii * 128 + ((rc ^ (ii & 7)) << 4) + rb) = __float2bfloat16_rn(ddv[u]);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // ---- Delta^T = Y^T A2^T ;  dY^T = dDelta^T A2 ;  [dDelta; dO] [Y^T | Delta^T] needs Delta^T: later
  if (tid == 0 && ok) {
    tc_fence_after();
    constexpr uint32_t id64 = idesc_bf16(128, 64, false, false);
    constexpr uint32_t idmm = idesc_bf16(128, 64, true, true);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      umma_f16(tmem + kColDt, kdesc(sbase + kOffYt + ks * 32), kdesc(sbase + kOffA2 + ks * 32), id64, ks > 0);
      // A[m=r][k=i] = dDelta[i][r]: token-major dD tile read MN-major (dv halves 16KB apart)
      umma_f16(tmem + kColDb, mdesc(sbase + kOffVDO + ks * 2048, 16384), mdesc(sbase + kOffA2 + ks * 2048, 8192), idmm,
               ks > 0);
    }
  }
  commit_wait();
  // ---- Delta^T -> bf16; dY^T -> dv (output) and -e^gam dY^T (bf16); dgam terms (1)-(4)
  float dgpart[32];
  {
    float dl[32], dy[32], sk[32], sq[32], da[32];
    if (ok) {
      tmem_ld32_sync(tmem + lane_base + kColDt + hh * 32, dl);
      tmem_ld32_sync(tmem + lane_base + kColDb + hh * 32, dy);
      tmem_ld32_sync(tmem + lane_base + kColY + hh * 32, sk);
      tmem_ld32_sync(tmem + lane_base + kColSQ + hh * 32, sq);
      tmem_ld32_sync(tmem + lane_base + kColDa + hh * 32, da);
    } else {
#pragma unroll
      for (int u = 0; u < 32; ++u) dl[u] = dy[u] = sk[u] = sq[u] = da[u] = 0.f;
    }
    const uint8_t* dot = sm + kOffVDO + 8192 + (r >> 6) * 16384;   // dO, token-major
    const int rc = (r & 63) >> 3, rb = (r & 7) * 2;
    float sj[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int jj = hh * 32 + u;
      const float dov = bf16_at(dot + jj * 128 + ((rc ^ (jj & 7)) << 4) + rb);
      // (1) + (2): scale e^gam_j dO_jr (S Q^T)_rj - e^gam_j dY_jr (S K^T)_rj
      if (kNorm) dgpart[u] = p.scale * dov * sq[u] * egq[jj] - dy[u] * sk[u] * egk[jj];
      else dgpart[u] = eg[jj] * (p.scale * dov * sq[u] - dy[u] * sk[u]);
      sj[u] = egd[jj] * dl[u] * da[u];                 // (3) s_j partial
    }
    uint32_t w[16], x[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      w[u] = pack_bf16(dl[2 * u], dl[2 * u + 1]);
      const int j0 = hh * 32 + 2 * u;
      x[u] = pack_bf16(-dy[2 * u] * egk[j0], -dy[2 * u + 1] * egk[j0 + 1]);
    }
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      st_shared_v4(sbase + kOffDt + sw128(r, hh * 4 + c4), w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
    }
    // the stacked product below still reads Y^T: -e^gam dY^T goes in after it
    // dv (token-major) from dY^T. A full chunk is staged as two 128B-swizzled 64-column halves
    // in the A2 / P slots (their products have completed) for two TMA tile stores after the
    // barrier below; a partial one is stored per thread (rows past the end are other data).
    if (nv == kChunk) {
      uint8_t* stg = sm + kOffA2 + (r >> 6) * 8192 + (r & 7) * 2;
      const int rc = (r & 63) >> 3;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int i = hh * 32 + u;
        *reinterpret_cast<__nv_bfloat16*>(stg + i * 128 + ((rc ^ (i & 7)) << 4)) = __float2bfloat16_rn(dy[u]);
      }
    } else if (ok) {
      __nv_bfloat16* dvo = static_cast<__nv_bfloat16*>(out.dv);
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int jj = hh * 32 + u;
        if (jj < nv) dvo[((size_t)(row + jj) * p.Hv + j) * 128 + r] = __float2bfloat16_rn(dy[u]);
      }
    }
    // reductions over r (the 128 TMEM lanes = 4 warps x 32 lanes) into per-token sums
    const float tot1 = warp_transpose_sum(dgpart);       // lane l: token hh*32 + l
    const float tot3 = warp_transpose_sum(sj);
    ss->dgam[kSlotTok + qd][hh * 32 + lane] = tot1 - tot3;
    float sred = tot3;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sred += __shfl_xor_sync(0xffffffffu, sred, off);
    if (lane == 0) ss->dgn[warp] = sred;                 // (3): sum_j s_j -> gam_n
    // keep -e^gam dY^T for later (registers -> written after the stacked product)
#pragma unroll
    for (int u = 0; u < 16; ++u) dgpart[u] = __uint_as_float(x[u]);
  }
  // (4) e^gam_n <S, dS'> over this thread's 64 entries (row r, half hh)
  {
    const uint8_t* sr = sm + kOffS + hh * 16384;
    const uint8_t* dsr = sm + kOffDS + hh * 16384;
    float acc = 0.f;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const uint4 a = *reinterpret_cast<const uint4*>(sr + sw128(r, ch));
      const uint4 d = *reinterpret_cast<const uint4*>(dsr + sw128(r, ch));
      const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* dh = reinterpret_cast<const __nv_bfloat162*>(&d);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 af = __bfloat1622float2(ah[e]), df = __bfloat1622float2(dh[e]);
        acc = fmaf(af.x, df.x, fmaf(af.y, df.y, acc));
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) ss->dgn[8 + warp] = ss->cs.egn[0] * acc;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // ---- [dDelta; dO] [Y^T | Delta^T]: rows 0..63 x cols 0..63 = dA2, rows 64..127 x cols 64..127 = dP / scale
  if (tid == 0 && ok && nv == kChunk) {       // dv tile stores (the staging is fenced above)
    tma_store_3d(&tm_dv, sbase + kOffA2, 0, j, row);
    tma_store_3d(&tm_dv, sbase + kOffA2 + 8192u, 64, j, row);
    bulk_commit();
  }
  if (tid == 0 && ok) {
    tc_fence_after();
    constexpr uint32_t id = idesc_bf16(128, 128, false, true);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t off = (ks >> 2) * 16384u + (ks & 3) * 32u;
      // B[k=r][n]: Y^T (n < 64) and Delta^T (n >= 64), tiles 16KB apart; k-step = 16 rows r
      umma_f16(tmem + kColD, kdesc(sbase + kOffVDO + off), mdesc(sbase + kOffYt + ks * 2048, 16384), id, ks > 0);
    }
  }
  if (tid == 0) bulk_wait_read();             // the P slot is rewritten (dPm) after this barrier
  commit_wait();
  // Y^T is free: -e^gam dY^T; Delta^T -> e^(gam_n - gam) Delta^T in place (dP has consumed it)
  {
    uint32_t x[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) x[u] = __float_as_uint(dgpart[u]);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
      st_shared_v4(sbase + kOffYt + sw128(r, hh * 4 + c4), x[4 * c4], x[4 * c4 + 1], x[4 * c4 + 2], x[4 * c4 + 3]);
    uint8_t* dtr = sm + kOffDt;
    uint4 q4[4];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) q4[c4] = *reinterpret_cast<const uint4*>(dtr + sw128(r, hh * 4 + c4));
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q4[c4]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int jj = hh * 32 + c4 * 8 + 2 * e;
        const float2 f = __bfloat1622float2(h[e]);
        h[e] = __floats2bfloat162_rn(f.x * egd[jj], f.y * egd[jj + 1]);
      }
      *reinterpret_cast<uint4*>(dtr + sw128(r, hh * 4 + c4)) = q4[c4];
    }
  }
  // ---- C x C step. Lanes 0..63 (quadrants 0, 1): row i of dA2 (cols 0..63) and of K K^T (G);
  //      lanes 64..127 (quadrants 2, 3): row i of dP (cols 64..127) and of Q K^T (G).
  {
    const int i = r & 63;
    float gvals[32], mvals[32];
    if (ok) {
      tmem_ld32_sync(tmem + lane_base + kColG + hh * 32, gvals);
      tmem_ld32_sync(tmem + lane_base + kColD + (r >= 64 ? 64 : 0) + hh * 32, mvals);
    } else {
#pragma unroll
      for (int u = 0; u < 32; ++u) gvals[u] = mvals[u] = 0.f;
    }
    // E_ij for this row's 32 columns by running products (as in the prep)
    const int j0 = hh * 32;
    float e[32];
    {
      const float gi = ss->cs.gam[0][i], glast = ss->cs.gam[0][j0 + 31];
      float run = 1.f;
#pragma unroll
      for (int jj = 31; jj >= 0; --jj) {
        const int jx = j0 + jj;
        if (jj == 31) run = (jx >= i) ? 1.f : fast_exp(gi - glast);
        else run = (jx >= i) ? 1.f : run * ss->cs.egt[0][jx + 1];
        e[jj] = run;
      }
    }
    const float* Lf = reinterpret_cast<const float*>(sm + kOffLf);   // A (fp32)
    float rowsum = 0.f;
    float colv[32];
    if (r < 64) {
      // dbeta_j += sum_i dA2_ij A_ij ;  dA = dA2 diag(beta) -> bf16
      const float* bet = ss->cs.bet[0];
      uint32_t w[16];
      {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 t = *reinterpret_cast<const float4*>(Lf + i * kChunk + a_chunk(i, (j0 >> 2) + u) * 4);
          colv[4 * u] = mvals[4 * u] * t.x;
          colv[4 * u + 1] = mvals[4 * u + 1] * t.y;
          colv[4 * u + 2] = mvals[4 * u + 2] * t.z;
          colv[4 * u + 3] = mvals[4 * u + 3] * t.w;
        }
      }
#pragma unroll
      for (int u = 0; u < 16; ++u)
        w[u] = pack_bf16(mvals[2 * u] * bet[j0 + 2 * u], mvals[2 * u + 1] * bet[j0 + 2 * u + 1]);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        st_shared_v4(sbase + kOffDA + sw128(i, hh * 4 + c4), w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
      const float cs_ = warp_transpose_sum(colv);
      ss->dbeta[kSlotBetaA + qd][j0 + lane] = cs_;       // qd in {0, 1}
    } else {
      // dP = scale * mvals;  P = QK^T * E (j <= i);  F = dP * P -> dgam_i += row sum, dgam_j -= col sum
      // dPm = dP * E (j <= i) -> bf16
      uint32_t w[16];
      if (kNorm) {                            // normalised P and dPm: rows times rq_i, columns times rk_j
        const float rqi = ss->cs.rq[0][i];
#pragma unroll
        for (int u = 0; u < 32; ++u) e[u] *= rqi * ss->cs.rk[0][j0 + u];
      }
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int jx = j0 + u;
        const bool m = jx <= i;
        const float dp = p.scale * mvals[u];
        const float pv = m ? gvals[u] * e[u] : 0.f;
        const float f = dp * pv;
        rowsum += f;
        colv[u] = f;
        mvals[u] = m ? dp * e[u] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) w[u] = pack_bf16(mvals[2 * u], mvals[2 * u + 1]);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        st_shared_v4(sbase + kOffP + sw128(i, hh * 4 + c4), w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
      const float cs_ = warp_transpose_sum(colv);
      ss->dgam[kSlotFP + (qd - 2)][j0 + lane] = -cs_;   // qd in {2, 3}
      ss->dgam[kSlotFPRow + hh][i] = rowsum;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // ---- X = dA A^T (rows i < 64 valid)
  if (tid == 0 && ok) {
    tc_fence_after();
    constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      umma_f16(tmem + kColDa, kdesc(sbase + kOffDA + ks * 32), kdesc(sbase + kOffA + ks * 32), id, ks > 0);
  }
  commit_wait();
  if (r < 64) {
    float xv[32];
    if (ok) tmem_ld32_sync(tmem + lane_base + kColDa + hh * 32, xv);
    else {
#pragma unroll
      for (int u = 0; u < 32; ++u) xv[u] = 0.f;
    }
    uint32_t w[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) w[u] = pack_bf16(xv[2 * u], xv[2 * u + 1]);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
      st_shared_v4(sbase + kOffDA + sw128(r, hh * 4 + c4), w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
  } else {
    // dO <- scale diag(e^gam) dO in place (an operand of dQ; times rq under the normalisation);
    // its other uses have completed
    scale_rows_tile_part(sm + kOffVDO + 8192, 16384, egq, p.scale, (r - 64) + 64 * hh, 128);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // ---- dL = -A^T X  (A read MN-major: A^T[i][k] = A[k][i]), then, behind it, every product of
  //      dQ = (scale e^gam dO) S + dPm K  and  dK = dPm^T Q + (-e^gam dY) S + (e^(gam_n-gam) Delta) dS'
  //      whose operands are ready (dK's dGs K term follows once dGs is written). They are issued by
  //      warp 2, which has no rows in the dL phase, so that the issue and the tensor-core time
  //      overlap that phase; only the threads of rows i < 64 wait for dL.
  if (tid == kLateIssuer && ok) {
    tc_fence_after();
    constexpr uint32_t id = idesc_bf16(128, 64, true, true);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      umma_f16(tmem + kColDb, mdesc(sbase + kOffA + ks * 2048, 8192), mdesc(sbase + kOffDA + ks * 2048, 8192), id,
               ks > 0);
    umma_commit(&ss->mma_bar);
    constexpr uint32_t idkm = idesc_bf16(128, 128, false, true);   // A K-major, B MN-major
    constexpr uint32_t idmm = idesc_bf16(128, 128, true, true);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t off = (ks >> 2) * 16384u + (ks & 3) * 32u;   // dO rows (K = r), 16 per step
      umma_f16(tmem + kColQ, kdesc(sbase + kOffVDO + 8192 + off), mdesc(sbase + kOffS + ks * 2048, 16384), idkm,
               ks > 0);
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      umma_f16(tmem + kColQ, kdesc(sbase + kOffP + ks * 32), mdesc(sbase + kOffKQ + ks * 2048, 16384), idkm, 1);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      umma_f16(tmem + kColK, mdesc(sbase + kOffP + ks * 2048, 8192), mdesc(sbase + kOffKQ + 8192 + ks * 2048, 16384),
               idmm, ks > 0);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      umma_f16(tmem + kColK, mdesc(sbase + kOffYt + ks * 2048, 16384), mdesc(sbase + kOffS + ks * 2048, 16384), idmm, 1);
      umma_f16(tmem + kColK, mdesc(sbase + kOffDt + ks * 2048, 16384), mdesc(sbase + kOffDS + ks * 2048, 16384), idmm,
               1);
    }
  }
  if (warp == 3) {
    // warp 3 has no rows in the dL phase: it finds this CTA's next item and forms its gate scalars in
    // slot 1 (the same arithmetic as prep_store_gb, prep_scan and prep_decays, two tokens per lane),
    // so that the next item starts with its loads
    int nx = item + gridDim.x;
    Pos np;
    while (nx < num_items && !decode_warp(nx, n, np)) nx += gridDim.x;
    int nrow = 0, nhq = 0, nsrow = 0;
    if (nx < num_items) {
      item_rows(np, nrow, nhq, nsrow);
      const int nnv = min(kChunk, np.e0 - (np.s0 + np.c * kChunk));
      const int so = 1, i0 = 2 * lane, i1 = 2 * lane + 1;
      float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
      const size_t gi = (size_t)nrow * p.Hv + np.j + (size_t)i0 * p.Hv;
      if (i0 < nnv) {
        a0 = p.g[gi];
        b0 = __bfloat162float(beta[gi]);
      }
      if (i1 < nnv) {
        a1 = p.g[gi + p.Hv];
        b1 = __bfloat162float(beta[gi + p.Hv]);
      }
      ss->cs.bet[so][i0] = b0;
      ss->cs.bet[so][i1] = b1;
      ss->cs.egt[so][i0] = fast_exp(a0);
      ss->cs.egt[so][i1] = fast_exp(a1);
      const float pair = a0 + a1;
      float run = pair;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, run, off);
        if (lane >= off) run += y;
      }
      const float gam0 = run - pair + a0, gam1 = run;
      const float gn = __shfl_sync(0xffffffffu, run, 31);
      ss->cs.gam[so][i0] = gam0;
      ss->cs.gam[so][i1] = gam1;
      ss->cs.eg[so][i0] = fast_exp(gam0);
      ss->cs.eg[so][i1] = fast_exp(gam1);
      ss->cs.egd[so][i0] = fast_exp(gn - gam0);
      ss->cs.egd[so][i1] = fast_exp(gn - gam1);
      if (lane == 0) {
        ss->cs.egn[so] = fast_exp(gn);
        ss->cs.nv[so] = nnv;
      }
    }
    if (lane == 0) {
      ss->next[0] = min(nx, num_items);
      ss->next[1] = np.n;
      ss->next[2] = np.c;
      ss->next[3] = np.j;
      ss->next[4] = np.b;
      ss->next[5] = np.s0;
      ss->next[6] = np.e0;
      ss->next[7] = nrow;
      ss->next[8] = nhq;
      ss->next[9] = nsrow;
    }
  }
  if (r < 64) {
    ok = ok && mbar_wait(&ss->mma_bar, mph, abort_flag);
    tc_fence_after();
  }
  mph ^= 1;
  // ---- dL (rows i < 64): strictly lower part. F += dL * L, dbeta_i += sum_j dL_ij KK_ij E_ij,
  //      dG = dL beta_i E (fp32 to Lf), then dGs = dG + dG^T -> bf16 (A's slot)
  {
    const int i = r & 63;
    const int j0 = hh * 32;
    float* Lf = reinterpret_cast<float*>(sm + kOffLf);
    if (r < 64) {
      float dlv[32], gvals[32];
      if (ok) {
        tmem_ld32_sync(tmem + lane_base + kColDb + hh * 32, dlv);
        tmem_ld32_sync(tmem + lane_base + kColG + hh * 32, gvals);
      } else {
#pragma unroll
        for (int u = 0; u < 32; ++u) dlv[u] = gvals[u] = 0.f;
      }
      const float gi = ss->cs.gam[0][i], glast = ss->cs.gam[0][j0 + 31];
      const float bi = ss->cs.bet[0][i];
      const float rki = kNorm ? ss->cs.rk[0][i] : 1.f;
      float run = 1.f, rowsum = 0.f, bsum = 0.f;
      float colv[32], dg[32];
#pragma unroll
      for (int jj = 31; jj >= 0; --jj) {
        const int jx = j0 + jj;
        if (jj == 31) run = (jx >= i) ? 1.f : fast_exp(gi - glast);
        else run = (jx >= i) ? 1.f : run * ss->cs.egt[0][jx + 1];
        const bool m = jx < i;
        const float dl = m ? -dlv[jj] : 0.f;
        // (K K^T)_ij E_ij of the normalised rows under the normalisation
        const float ke = kNorm ? gvals[jj] * run * (rki * ss->cs.rk[0][jx]) : gvals[jj] * run;
        const float f = dl * bi * ke;            // dL * L
        rowsum += f;
        colv[jj] = f;
        bsum += dl * ke;
        dg[jj] = dl * bi * run;
      }
      // A (fp32) in Lf has no readers left: dG takes its place
      {
        float4* dst = reinterpret_cast<float4*>(Lf + i * kLd + j0);
#pragma unroll
        for (int u = 0; u < 8; ++u) dst[u] = make_float4(dg[4 * u], dg[4 * u + 1], dg[4 * u + 2], dg[4 * u + 3]);
      }
      const float cs_ = warp_transpose_sum(colv);
      ss->dgam[kSlotFL + qd][j0 + lane] = -cs_;         // qd in {0, 1}
      ss->dgam[kSlotFLRow + hh][i] = rowsum;
      // bsum: this thread's half of row i; the other half is in warp qd + 4
      ss->dbeta[kSlotBetaL + hh][i] = bsum;
    }
  }
  __syncthreads();
  if (r < 64) {
    const int i = r, j0 = hh * 32;
    const float* Lf = reinterpret_cast<const float*>(sm + kOffLf);
    uint32_t w[16];
    const float4* rowv = reinterpret_cast<const float4*>(Lf + i * kLd + j0);
    if (kNorm) {                              // dGs multiplies the raw K: rk_i (dG + dG^T)_ij rk_j
      const float rki = ss->cs.rk[0][i];
      const float* rk = ss->cs.rk[0];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 t = rowv[u];
        const int ja = j0 + 4 * u;
        w[2 * u] = pack_bf16((t.x + Lf[ja * kLd + i]) * rki * rk[ja], (t.y + Lf[(ja + 1) * kLd + i]) * rki * rk[ja + 1]);
        w[2 * u + 1] = pack_bf16((t.z + Lf[(ja + 2) * kLd + i]) * rki * rk[ja + 2],
                                 (t.w + Lf[(ja + 3) * kLd + i]) * rki * rk[ja + 3]);
      }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 t = rowv[u];
        const int ja = j0 + 4 * u;
        w[2 * u] = pack_bf16(t.x + Lf[ja * kLd + i], t.y + Lf[(ja + 1) * kLd + i]);
        w[2 * u + 1] = pack_bf16(t.z + Lf[(ja + 2) * kLd + i], t.w + Lf[(ja + 3) * kLd + i]);
      }
    }
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
      st_shared_v4(sbase + kOffA + sw128(i, hh * 4 + c4), w[4 * c4], w[4 * c4 + 1], w[4 * c4 + 2], w[4 * c4 + 3]);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // ---- dK += dGs K (same issuing thread as the rest of dK)
  if (tid == kLateIssuer && ok) {
    tc_fence_after();
    constexpr uint32_t idkm = idesc_bf16(128, 128, false, true);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      umma_f16(tmem + kColK, kdesc(sbase + kOffA + ks * 32), mdesc(sbase + kOffKQ + ks * 2048, 16384), idkm, 1);
  }
  commit_wait(kLateIssuer);
  {
    const int pnx = ss->next[0];
    prefetched = ok && pnx < num_items;
    if (prefetched) {
      const int nrow = ss->next[7], nhq = ss->next[8], nsrow = ss->next[9];
      if (tid == kLateIssuer) {
        mbar_arrive_expect_tx(&ss->tma_bar, kItemBytes);
        if (!kNorm) load_kq(nhq, nrow);
        load_rest(ss->next[3], nrow, nsrow);
        load_ap(nsrow);
      }
    }
  }
  // ---- outputs: dq, dk (rows i < nv), dbeta, dg. A full chunk's bf16 dq, dk leave through TMA
  //      tile stores from staging (every operand tile is free now), otherwise per thread.
  const bool qk_tma = !out.qk_partial && nv == kChunk;
  // Under the normalisation the accumulators hold x = r * (gradient w.r.t. the normalised row); the
  // gradient w.r.t. the raw row is x - xn (xn . x), xn = r * (raw row). This thread holds 64 of
  // the row's 128 columns (the other half is in warp qd + 4): partial dot products through smem.
  // raw_half: row i, column half hh of the Q (which = 0) or K (which = 1) tile (bf16, swizzled)
  auto raw_half = [&](int which, int i) -> const uint8_t* {
    return sm + kOffKQ + (which == 0 ? 8192 : 0) + hh * 16384 + i * 128;
  };
  if (kNorm) {
    if (r < 64) {
      const int i = r;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        float v[64];
        const uint32_t col = which == 0 ? kColQ : kColK;
        if (ok) {
          tmem_ld32_sync(tmem + lane_base + col + hh * 64, v);
          tmem_ld32_sync(tmem + lane_base + col + hh * 64 + 32, v + 32);
        } else {
#pragma unroll
          for (int u = 0; u < 64; ++u) v[u] = 0.f;
        }
        const uint8_t* xr = raw_half(which, i);
        float acc = 0.f;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xr + ((ch ^ (i & 7)) << 4));
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float2 f = __bfloat1622float2(h2[e2]);
            acc = fmaf(f.x, v[8 * ch + 2 * e2], fmaf(f.y, v[8 * ch + 2 * e2 + 1], acc));
          }
        }
        ss->pdot[which][hh][i] = acc;
      }
    }
    __syncthreads();
  }
  if (r < 64) {
    const int i = r;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      float v[64];
      const uint32_t col = which == 0 ? kColQ : kColK;
      if (ok) {
        tmem_ld32_sync(tmem + lane_base + col + hh * 64, v);
        tmem_ld32_sync(tmem + lane_base + col + hh * 64 + 32, v + 32);
      }
      if (kNorm && ok) {
        // v -= xn (xn . v) = raw * (r^2 (raw . v)), both halves summed in a fixed order
        const float ri = which == 0 ? ss->cs.rq[0][i] : ss->cs.rk[0][i];
        const float coef = ri * ri * (ss->pdot[which][0][i] + ss->pdot[which][1][i]);
        const uint8_t* xr = raw_half(which, i);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xr + ((ch ^ (i & 7)) << 4));
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float2 f = __bfloat1622float2(h2[e2]);
            v[8 * ch + 2 * e2] = fmaf(-coef, f.x, v[8 * ch + 2 * e2]);
            v[8 * ch + 2 * e2 + 1] = fmaf(-coef, f.y, v[8 * ch + 2 * e2 + 1]);
          }
        }
      }
      if (qk_tma) {                            // staged: Yt (dq) / Dt (dk), 128B-swizzled halves
        uint8_t* srow = sm + (which == 0 ? kOffYt : kOffDt) + hh * 8192 + i * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<uint4*>(srow + ((u ^ (i & 7)) << 4)) =
              make_uint4(pack_bf16(v[8 * u], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
                         pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
      } else if (ok && i < nv) {
        if (out.qk_partial) {                  // grouped values: fp32 per v-head, summed later
          float* dst = (which == 0 ? out.dq_part : out.dk_part) + ((size_t)(row + i) * p.Hv + j) * 128 + hh * 64;
#pragma unroll
          for (int u = 0; u < 16; ++u)
            reinterpret_cast<float4*>(dst)[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
        } else {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(which == 0 ? out.dq : out.dk) +
                               ((size_t)(row + i) * p.Hqk + hq) * 128 + hh * 64;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            reinterpret_cast<uint4*>(dst)[u] =
                make_uint4(pack_bf16(v[8 * u], v[8 * u + 1]), pack_bf16(v[8 * u + 2], v[8 * u + 3]),
                           pack_bf16(v[8 * u + 4], v[8 * u + 5]), pack_bf16(v[8 * u + 6], v[8 * u + 7]));
        }
      }
    }
  }
  if (qk_tma) {
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0 && ok) {
      tma_store_3d(&tm_dq, sbase + kOffYt, 0, hq, row);
      tma_store_3d(&tm_dq, sbase + kOffYt + 8192u, 64, hq, row);
      tma_store_3d(&tm_dk, sbase + kOffDt, 0, hq, row);
      tma_store_3d(&tm_dk, sbase + kOffDt + 8192u, 64, hq, row);
      bulk_commit();
    }
  }
  // warp 2 (no dq / dk rows above) turns the per-token slots into dg, dbeta while the
  // others store dq, dk; every slot was written before the last product's barrier
  if (warp == 2) {
    // dgam_{63} += dgn; dg = reverse cumsum of dgam over the chunk (two values per lane)
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int sl = 0; sl < kNumGamSlots; ++sl) {
      a0 += ss->dgam[sl][2 * lane];
      a1 += ss->dgam[sl][2 * lane + 1];
    }
    if (lane == 31) {
      float gn = 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u) gn += ss->dgn[u];
      a1 += gn;
    }
    float b0 = 0.f, b1 = 0.f;
#pragma unroll
    for (int sl = 0; sl < kNumBetaSlots; ++sl) {
      b0 += ss->dbeta[sl][2 * lane];
      b1 += ss->dbeta[sl][2 * lane + 1];
    }
    // reverse inclusive scan: dg_t = sum_{i >= t} dgam_i
    const float pair = a0 + a1;
    float run = pair;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_down_sync(0xffffffffu, run, off);
      if (lane + off < 32) run += y;
    }
    const float dg1 = run - a0;              // sum from 2*lane+1 up
    const float dg0 = run;                   // sum from 2*lane up
    if (ok) {
      const size_t gi = (size_t)(row + 2 * lane) * p.Hv + j;
      if (2 * lane < nv) out.dg[gi] = dg0;
      if (2 * lane + 1 < nv) out.dg[gi + p.Hv] = dg1;
      __nv_bfloat16* db = static_cast<__nv_bfloat16*>(out.dbeta);
      if (2 * lane < nv) db[gi] = __float2bfloat16_rn(b0);
      if (2 * lane + 1 < nv) db[gi + p.Hv] = __float2bfloat16_rn(b1);
    }
  }
  // the next item's loads overwrite every tile and TMEM column this one used
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  item = ss->next[0];
  pos = Pos{ss->next[1], ss->next[2], ss->next[3], ss->next[4], ss->next[5], ss->next[6]};
  scal_ready = true;
  }
  if (tid == 0) bulk_wait_all();
  if (tid == 0 && *abort_flag) {
    volatile int never = 0;
    mbar_wait(&ss->tma_bar, prefetched ? tph : (tph ^ 1), &never);
    report_error(p, kDevTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// fp32 per-v-head partials of dq / dk -> the sum over the v-heads of each q/k head (fixed order)
__global__ void gdn_bwd_reduce_kernel(const float* part, __nv_bfloat16* dst, int rows, int Hv, int Hqk) {
  const int group = Hv / Hqk;
  const size_t total = (size_t)rows * Hqk * 128;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (size_t)gridDim.x * blockDim.x) {
    const size_t d = idx % 128;
    const size_t h = (idx / 128) % Hqk;
    const size_t t = idx / (128 * Hqk);
    float acc = 0.f;
    for (int g = 0; g < group; ++g) acc += part[(t * Hv + h * group + g) * 128 + d];
    dst[idx] = __float2bfloat16_rn(acc);
  }
}

// [slots * 128, 128] bf16 state array: boxes of 128 rows x 64 columns, 128B swizzle
static bool make_state_map(CUtensorMap* m, const void* base, long long slots) {
  return make_tile_map(m, base, 1, slots * 128, 128);
}

cudaError_t launch_bwd_grad(const FwdParams& p, const BwdOut& out, long long total_chunks, cudaStream_t st,
                            const char** what) {
  if (total_chunks <= 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, mdo, ms, mds;
  const long long rows = (long long)p.B * p.T;
  *what = "tensor map encode";
  if (!make_tile_map(&mq, p.q, p.Hqk, rows) || !make_tile_map(&mk, p.k, p.Hqk, rows) ||
      !make_tile_map(&mv, p.v, p.Hv, rows) || !make_tile_map(&mdo, out.dO, p.Hv, rows) ||
      !make_state_map(&ms, p.states, total_chunks * p.Hv) || !make_state_map(&mds, out.dstates, total_chunks * p.Hv))
    return cudaErrorInvalidValue;
  CUtensorMap mdv, mdq = mq, mdk = mq;       // dq, dk maps only for the bf16 (non-grouped) outputs
  if (!make_tile_map(&mdv, out.dv, p.Hv, rows)) return cudaErrorInvalidValue;
  if (!out.qk_partial && (!make_tile_map(&mdq, out.dq, p.Hqk, rows) || !make_tile_map(&mdk, out.dk, p.Hqk, rows)))
    return cudaErrorInvalidValue;
  *what = "shared memory attribute";
  auto kernel = p.qk_l2norm ? gdn_bwd_grad_kernel<true> : gdn_bwd_grad_kernel<false>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (err != cudaSuccess) return err;
  // persistent: one CTA per SM (the shared-memory footprint allows one), items strided over CTAs
  const long long items = total_chunks * p.Hv;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  *what = "device query";
  err = cudaGetDevice(&dev);
  if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (err != cudaSuccess) return err;
  const unsigned grid = (unsigned)std::min<long long>(items, std::max(sms, 1));
  *what = "backward gradient launch";
  trace_pre(kKernBwdTc, st);
  kernel<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, mdo, ms, mds, mdv, mdq, mdk, p, out, (int)items);
  err = cudaGetLastError();
  trace_post(st);
  if (err != cudaSuccess || !out.qk_partial) return err;
  *what = "backward dq/dk reduction";
  const int rows_i = p.B * p.T;
  const int blocks = (int)std::min<long long>(4096, ((long long)rows_i * p.Hqk * 128 + 255) / 256);
  trace_pre(kKernBwdReduce, st);
  gdn_bwd_reduce_kernel<<<blocks, 256, 0, st>>>(out.dq_part, static_cast<__nv_bfloat16*>(out.dq), rows_i, p.Hv, p.Hqk);
  gdn_bwd_reduce_kernel<<<blocks, 256, 0, st>>>(out.dk_part, static_cast<__nv_bfloat16*>(out.dk), rows_i, p.Hv, p.Hqk);
  err = cudaGetLastError();
  trace_post(st);
  return err;
}

}  // namespace gdn
