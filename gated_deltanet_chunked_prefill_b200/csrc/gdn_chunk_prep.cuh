// State-independent per-chunk work shared by the tensor-core kernels (forward, the
// backward's reverse state-gradient chain, the backward's gradient kernel), for one
// 64-token chunk of one (sequence, v-head), run by a group of 256 threads (8 warps;
// warp w reads TMEM lane quadrant w % 4 and column half w / 4):
//
//   gam = inclusive cumsum of g,  E_ij = exp(gam_i - gam_j)
//   G = [K;Q] K^T   (one tcgen05 product, rows 0..63 = K K^T, rows 64..127 = Q K^T)
//   L = strict_lower(diag(beta) K K^T * E)  -> fp16;  A = (I + L)^-1: 16 x 16 diagonal
//       blocks by substitution, then 2 x 2 blocking into 32 x 32 blocks (m16n8k16 products)
//   P = lower_incl(Q K^T * E) * p_scale     -> bf16
//   A2 = A diag(beta) -> bf16 (with B2 = A diag(beta exp(gam)), or A in bf16 and fp32)
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "gdn_common.cuh"
#include "tc_ptx.cuh"

namespace gdn {

// Row stride (floats) of the fp32 64 x 64 scratch rows (A and dG in the gradient kernel).
// 68: row-per-thread accesses go through 16-byte vectors (8 threads per phase, rows 4 banks
// apart: conflict-free) and column-per-thread accesses stay scalar (consecutive rows,
// distinct banks).
constexpr int kLd = 68;
// Row stride (halves) of the fp16 64 x 64 variant of the scratch: 36 words = 4 mod 32, so
// the m16n8k16 A fragments (row gid, word tig) hit 32 distinct banks.
constexpr int kLdh = 72;
constexpr int kPrepThreads = 256;

// Layout of a stored A (fp32 64 x 64): row i, 16-byte chunk k of the row at chunk k ^ (i % 16),
// so that a strip's fragment writes hit distinct banks; the whole 16 KB moves as one copy.
__device__ __forceinline__ int a_chunk(int row, int k) { return k ^ (row & 15); }

// per-chunk scalars, double-buffered by chunk parity
struct ChunkScalars {
  float gam[2][64];   // chunk-local inclusive cumsum of g
  float egt[2][64];   // exp(g_t) (1 past the sequence end)
  float eg[2][64];    // exp(gam)
  float egd[2][64];   // exp(gam_n - gam), times rk under the q/k normalisation
  float bet[2][64];   // beta (0 past the sequence end)
  float egn[2];       // exp(gam_n)
  int nv[2];          // valid tokens in the chunk
  // q/k normalisation only: the inverse row norms (|x|^2 + eps)^(-1/2) of the chunk's K and Q
  // rows, and exp(gam) times them. A normalised row is r * (raw row), so every product with a
  // normalised K or Q row is the raw tile's product with r folded into a per-token factor.
  float rk[2][64], rq[2][64];
  float egk[2][64];   // exp(gam) rk
  float egq[2][64];   // exp(gam) rq
};

// eps of the in-kernel q/k normalisation x / sqrt(|x|^2 + eps)
constexpr float kL2NormEps = 1e-6f;

// Inverse row norms of a chunk's K and Q tiles in shared memory (64 rows x 128 bf16 each, held
// as two 64-column halves of 128-byte rows; the swizzle only permutes a row's 16-byte pieces).
// 256 threads, two per row: threads 0..127 take K rows, 128..255 Q rows.
__device__ __forceinline__ void row_inv_norms(const uint8_t* k0, const uint8_t* k1, const uint8_t* q0,
                                              const uint8_t* q1, float* rk, float* rq, int t) {
  const int row = (t >> 1) & 63, half = t & 1;
  const bool isq = t >= 128;
  const uint8_t* base = (isq ? (half ? q1 : q0) : (half ? k1 : k0)) + row * 128;
  float ssq = 0.f;
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    const uint4 v = *reinterpret_cast<const uint4*>(base + ch * 16);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      ssq = fmaf(f.x, f.x, fmaf(f.y, f.y, ssq));
    }
  }
  ssq += __shfl_xor_sync(0xffffffffu, ssq, 1);
  if (half == 0) (isq ? rq : rk)[row] = rsqrtf(ssq + kL2NormEps);
}

__device__ __forceinline__ float bf16_at(const uint8_t* p) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}

// 16-byte chunk of 8 bf16 values, scaled
__device__ __forceinline__ uint4 scale_chunk(uint4 v, float f) {
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 x = __bfloat1622float2(h[i]);
    h[i] = __floats2bfloat162_rn(x.x * f, x.y * f);
  }
  return v;
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

struct PrepCtx {
  uint32_t sbase;     // shared address of the 1024-aligned smem base
  float* Lf;          // scratch: fp16 L [64][kLdh]; fp32 rows [64][kLd] where a kernel asks
  ChunkScalars* cs;
  uint32_t tmem;      // TMEM base
  uint32_t colG;      // TMEM column of G
  int pt, pw, lane;   // thread index in the group, warp in the group, lane
  int bar;            // named barrier id of the group
};

// g, beta of the chunk -> scalars (step 1: before the scan). gv, bv are this thread's
// values (0 past the sequence end), loaded by the caller.
__device__ __forceinline__ void prep_store_gb(const PrepCtx& c, int s, float gv, float bv) {
  if (c.pt < kChunk) {
    c.cs->gam[s][c.pt] = gv;
    c.cs->bet[s][c.pt] = bv;
    c.cs->egt[s][c.pt] = tc::fast_exp(gv);
  }
}

// inclusive cumsum (warp 0) -- the caller separates this from prep_store_gb with a barrier
__device__ __forceinline__ void prep_scan(const PrepCtx& c, int s) {
  if (c.pw == 0) {
    const float a0 = c.cs->gam[s][2 * c.lane], a1 = c.cs->gam[s][2 * c.lane + 1];
    const float pair = a0 + a1;
    float run = pair;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, run, off);
      if (c.lane >= off) run += y;
    }
    c.cs->gam[s][2 * c.lane] = run - pair + a0;
    c.cs->gam[s][2 * c.lane + 1] = run;
  }
}

// decay factors (after the scan and a barrier; under the q/k normalisation also after the
// inverse row norms): eg, egd (times rk when kNorm), and with kNorm egk, egq
template <bool kNorm = false>
__device__ __forceinline__ void prep_decays(const PrepCtx& c, int s, int nv) {
  const float gn = c.cs->gam[s][kChunk - 1];
  if (c.pt < kChunk) {
    const float e = tc::fast_exp(c.cs->gam[s][c.pt]);
    const float ed = tc::fast_exp(gn - c.cs->gam[s][c.pt]);
    c.cs->eg[s][c.pt] = e;
    if (kNorm) {
      const float rk = c.cs->rk[s][c.pt];
      c.cs->egd[s][c.pt] = ed * rk;
      c.cs->egk[s][c.pt] = e * rk;
      c.cs->egq[s][c.pt] = e * c.cs->rq[s][c.pt];
    } else {
      c.cs->egd[s][c.pt] = ed;
    }
  }
  if (c.pt == 0) {
    c.cs->egn[s] = tc::fast_exp(gn);
    c.cs->nv[s] = nv;
  }
}

// Issue G = [K;Q] K^T and commit to `bar`. K0, Q0 (8KB sub-tiles, dk 0..63) are adjacent
// at kq_addr; K1, Q1 (dk 64..127) follow at kq_addr + half_stride.
__device__ __forceinline__ void issue_gram(uint32_t tmem_g, uint32_t kq_addr, uint64_t* bar,
                                           uint32_t half_stride = 16384u) {
  constexpr uint32_t id = tc::idesc_bf16(128, 64, false, false);
  tc::tc_fence_after();
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const uint32_t off = (ks >> 2) * half_stride + (ks & 3) * 32u;
    tc::umma_f16(tmem_g, tc::sdesc_sw128(kq_addr + off, 16, 1024), tc::sdesc_sw128(kq_addr + off, 16, 1024), id,
                 ks > 0);
  }
  tc::umma_commit(bar);
}

// G (TMEM) -> L (fp16 rows of stride kLdh in Lf, strictly lower) and P = p_scale * lower_incl(QK^T * E) (bf16,
// 128B-swizzled rows at p_addr). E_ij = exp(gam_i - gam_j) (j <= i) is the running product
// of exp(g_t) over t = j+1..i, walking j down: one exponential per row segment instead of
// one per entry, no overflow, monotone underflow to 0. `ok` false: G treated as 0.
// Ends with tcgen05 fence + group barrier.
// kWriteL false: only P is produced (the caller takes A from elsewhere).
// kNorm: G holds raw-row products; the normalised ones are rk_i rk_j (KK^T)_ij and
// rq_i rk_j (QK^T)_ij, so the rows take rk_i (L) or rq_i (P) and the columns rk_j.
template <bool kWriteL = true, bool kNorm = false>
__device__ __forceinline__ void prep_masks(const PrepCtx& c, int s, uint32_t p_addr, float p_scale, bool ok) {
  const int qd = c.pw & 3, hc = c.pw >> 2;
  const int rr = 32 * qd + c.lane;
  const int j0 = 32 * hc;
  float vals[32];
  if (ok) {
    tc::tmem_ld32_sync(c.tmem + ((uint32_t)(32 * qd) << 16) + c.colG + j0, vals);
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) vals[j] = 0.f;
  }
  float et[32];
  {
    const float4* e4 = reinterpret_cast<const float4*>(c.cs->egt[s] + j0);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 t = e4[u];
      et[4 * u] = t.x; et[4 * u + 1] = t.y; et[4 * u + 2] = t.z; et[4 * u + 3] = t.w;
    }
  }
  const int i = rr & 63;
  const float gi = c.cs->gam[s][i];
  const float glast = c.cs->gam[s][j0 + 31];
  if (kNorm) {
    const float4* r4 = reinterpret_cast<const float4*>(c.cs->rk[s] + j0);
    const float rowf = rr < kChunk ? c.cs->rk[s][i] : c.cs->rq[s][i];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 t = r4[u];
      vals[4 * u] *= rowf * t.x; vals[4 * u + 1] *= rowf * t.y;
      vals[4 * u + 2] *= rowf * t.z; vals[4 * u + 3] *= rowf * t.w;
    }
  }
  float run = 1.f;
  if (rr < kChunk && !kWriteL) {
    // L not wanted
  } else if (rr < kChunk) {
    const float bi = c.cs->bet[s][i];
#pragma unroll
    for (int jj = 31; jj >= 0; --jj) {
      const int j = j0 + jj;
      if (jj == 31) run = (j >= i) ? 1.f : tc::fast_exp(gi - glast);
      else run = (j >= i) ? 1.f : run * et[jj + 1];
      vals[jj] = (j < i) ? bi * vals[jj] * run : 0.f;
    }
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__half*>(c.Lf) + i * kLdh + j0);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      dst[u] = make_uint4(pack_h2(vals[8 * u], vals[8 * u + 1]), pack_h2(vals[8 * u + 2], vals[8 * u + 3]),
                          pack_h2(vals[8 * u + 4], vals[8 * u + 5]), pack_h2(vals[8 * u + 6], vals[8 * u + 7]));
  } else {
#pragma unroll
    for (int jj = 31; jj >= 0; --jj) {
      const int j = j0 + jj;
      if (jj == 31) run = (j >= i) ? 1.f : tc::fast_exp(gi - glast);
      else run = (j >= i) ? 1.f : run * et[jj + 1];
      vals[jj] = (j <= i) ? vals[jj] * run * p_scale : 0.f;
    }
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4)
      st_shared_v4(p_addr + tc::sw128(i, 4 * hc + c4), tc::pack_bf16(vals[c4 * 8 + 0], vals[c4 * 8 + 1]),
                   tc::pack_bf16(vals[c4 * 8 + 2], vals[c4 * 8 + 3]), tc::pack_bf16(vals[c4 * 8 + 4], vals[c4 * 8 + 5]),
                   tc::pack_bf16(vals[c4 * 8 + 6], vals[c4 * 8 + 7]));
  }
  tc::tc_fence_before();
  tc::named_bar_sync(c.bar, kPrepThreads);
}

// Scale rows of a [64 x 128] bf16 tile (two 8KB 128B-swizzled sub-tiles, sub-tile 1 at
// +sub_stride) by f[row] * mult, in place, with nt threads (t = this thread's index).
__device__ __forceinline__ void scale_rows_tile_part(uint8_t* tile, uint32_t sub_stride, const float* f, float mult,
                                                     int t, int nt) {
  for (int idx = t; idx < 1024; idx += nt) {
    const int row = idx >> 4, half = (idx >> 3) & 1, ch = idx & 7;
    uint4* q = reinterpret_cast<uint4*>(tile + half * sub_stride + row * 128 + ch * 16);
    *q = scale_chunk(*q, f[row] * mult);
  }
}

// ---- the inverse: L and the diagonal-block inverses D_R held as fp16 rows of stride kLdh
// (11-bit significand), the products below the diagonal on m16n8k16 f16 tensor instructions
// with fp32 accumulation.

// Diagonal 16 x 16 blocks, inverted in place (fp32 arithmetic, fp16 storage). Warps 0..3.
// af != nullptr: the blocks also go to af in fp32 (the stored-A layout, 64 x 64).
__device__ __forceinline__ void prep_diag_inverse_h(const PrepCtx& c, float* af = nullptr) {
  __half* Lh = reinterpret_cast<__half*>(c.Lf);
  const int R = c.pw, col = c.lane & 15;
  float a[16];
#pragma unroll
  for (int ii = 0; ii < 16; ++ii) {
    float l[16];
    const uint4* row = reinterpret_cast<const uint4*>(Lh + (16 * R + ii) * kLdh + 16 * R);
#pragma unroll
    for (int q8 = 0; q8 < (ii + 7) / 8; ++q8) {
      const uint4 t = row[q8];
      const __half2* h = reinterpret_cast<const __half2*>(&t);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        l[8 * q8 + 2 * e] = f.x;
        l[8 * q8 + 2 * e + 1] = f.y;
      }
    }
    float acc0 = (ii == col) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
    for (int jj = 0; jj < ii; jj += 2) {
      acc0 -= l[jj] * a[jj];
      if (jj + 1 < ii) acc1 -= l[jj + 1] * a[jj + 1];
    }
    a[ii] = (ii < col) ? 0.f : acc0 + acc1;
  }
  __syncwarp();
  if (c.lane < 16) {
#pragma unroll
    for (int ii = 0; ii < 16; ++ii) Lh[(16 * R + ii) * kLdh + 16 * R + col] = __float2half_rn(a[ii]);
    if (af != nullptr) {
      const int j = 16 * R + col;
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int i = 16 * R + ii;
        af[i * kChunk + a_chunk(i, j >> 2) * 4 + (j & 3)] = a[ii];
      }
    }
  }
}

__device__ __forceinline__ void mma_f16_16816(float* d, const uint32_t* a, const uint32_t* b) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// A fragment (16 x 16 at rows r0.., columns k0..) of the fp16 scratch: half pairs
__device__ __forceinline__ void lh_afrag(const __half* Lh, int r0, int k0, int gid, int tig, uint32_t* af) {
  const uint32_t* w0 = reinterpret_cast<const uint32_t*>(Lh + (r0 + gid) * kLdh + k0) + tig;
  const uint32_t* w1 = reinterpret_cast<const uint32_t*>(Lh + (r0 + gid + 8) * kLdh + k0) + tig;
  af[0] = w0[0];
  af[1] = w1[0];
  af[2] = w0[4];
  af[3] = w1[4];
}

// B fragment (k rows 0..15 of a 16 x 8 tile in accumulator layout) as fp16 pairs, by
// shuffles: b0 = rows 2 tig, 2 tig + 1 and b1 = rows 2 tig + 8, 2 tig + 9, at column gid.
__device__ __forceinline__ void acc_to_bfrag_h(const float* x, int lane, uint32_t* bf) {
  const int gid = lane >> 2, tig = lane & 3;
  const int sa = 8 * tig + (gid >> 1), sb = sa + 4;
  const bool odd = gid & 1;
  const float a0 = __shfl_sync(0xffffffffu, x[0], sa), a1 = __shfl_sync(0xffffffffu, x[1], sa);
  const float a2 = __shfl_sync(0xffffffffu, x[2], sa), a3 = __shfl_sync(0xffffffffu, x[3], sa);
  const float b0 = __shfl_sync(0xffffffffu, x[0], sb), b1 = __shfl_sync(0xffffffffu, x[1], sb);
  const float b2 = __shfl_sync(0xffffffffu, x[2], sb), b3 = __shfl_sync(0xffffffffu, x[3], sb);
  bf[0] = pack_h2(odd ? a1 : a0, odd ? b1 : b0);
  bf[1] = pack_h2(odd ? a3 : a2, odd ? b3 : b2);
}

// B fragment (k16 x n8, the "col" operand of m16n8k16) of the fp16 scratch: B[k][n] at rows k0 + k,
// columns n0 + n (b0 = rows 2 tig, 2 tig + 1; b1 = rows 2 tig + 8, 2 tig + 9; column gid)
__device__ __forceinline__ void lh_bfrag(const __half* Lh, int k0, int n0, int gid, int tig, uint32_t* bf) {
  const __half* p = Lh + (k0 + 2 * tig) * kLdh + n0 + gid;
  __half2 h0 = __halves2half2(p[0], p[kLdh]);
  __half2 h1 = __halves2half2(p[8 * kLdh], p[9 * kLdh]);
  bf[0] = *reinterpret_cast<uint32_t*>(&h0);
  bf[1] = *reinterpret_cast<uint32_t*>(&h1);
}

// fp32 accumulator fragment (16 x 8) -> the fp16 scratch (rows r0 + gid (+8), columns n0 + 2 tig (+1))
__device__ __forceinline__ void lh_store_acc(__half* Lh, int r0, int n0, int gid, int tig, const float* y) {
  *reinterpret_cast<__half2*>(Lh + (r0 + gid) * kLdh + n0 + 2 * tig) = __floats2half2_rn(y[0], y[1]);
  *reinterpret_cast<__half2*>(Lh + (r0 + gid + 8) * kLdh + n0 + 2 * tig) = __floats2half2_rn(y[2], y[3]);
}

// fp32 accumulator fragment (16 x 8) -> af (the stored-A layout), negated
__device__ __forceinline__ void af_store_neg_acc(float* af, int r0, int n0, int gid, int tig, const float* y) {
  const int j = n0 + 2 * tig;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = r0 + gid + 8 * h;
    *reinterpret_cast<float2*>(af + i * kChunk + a_chunk(i, j >> 2) * 4 + (j & 3)) = make_float2(-y[2 * h], -y[2 * h + 1]);
  }
}

// Zero the strictly upper 16 x 16 blocks of af (the stored-A layout), with nt threads.
__device__ __forceinline__ void af_zero_upper(float* af, int t, int nt) {
  // blocks (R, C), C > R: (0,1) (0,2) (0,3) (1,2) (1,3) (2,3); 16 rows x 4 16-byte pieces each
  for (int idx = t; idx < 6 * 64; idx += nt) {
    const int blk = idx >> 6, rem = idx & 63;
    const int R = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
    const int C = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
    const int i = 16 * R + (rem >> 2), k = 4 * C + (rem & 3);
    *reinterpret_cast<float4*>(af + i * kChunk + a_chunk(i, k) * 4) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// A = (I + L)^-1 below its 16 x 16 diagonal blocks D_R (already inverted in place in the fp16
// scratch and written to af by prep_diag_inverse_h), by 2 x 2 blocking into 32 x 32 blocks:
//   X10 = -D1 L10 D0,  X32 = -D3 L32 D2        (the 32 x 32 diagonal blocks A11, A22)
//   T   = L21 A11 = [L21a D0 + L21b X10 | L21b D1]   (L21 = [L21a | L21b], rows 32..63, cols 0..31)
//   A21 = -A22 T = -[D2 T_top ; X32 T_top + D3 T_bot]
// on m16n8k16 f16 products with fp32 accumulation: X10 / X32 on warps 0..3 (one 8-column tile
// each, two dependent products through shuffles), T on warps 4..7 (two tiles each), A21 on all
// eight (one tile each). X10, X32 replace L10, L32 in the scratch; T goes to its unused upper
// right 32 x 32 block (rows 0..31, columns 32..63). Every result goes to af in fp32. Three group
// barriers inside; the caller separates the last af writes from their readers with a barrier.
__device__ __forceinline__ void prep_inverse_blocked(const PrepCtx& c, float* af) {
  __half* Lh = reinterpret_cast<__half*>(c.Lf);
  const int w = c.pw, gid = c.lane >> 2, tig = c.lane & 3;
  float x[4] = {0.f, 0.f, 0.f, 0.f};        // warps 0..3: the X tile
  float ta[4] = {0.f, 0.f, 0.f, 0.f};       // warps 4..7: T tile in columns 0..15 (two terms)
  float tb[4] = {0.f, 0.f, 0.f, 0.f};       // warps 4..7: T tile in columns 16..31
  const int m = w & 3, tr = (m >> 1) * 16;  // warps 4..7: T rows tr .. tr + 15 (L rows 32 + tr ..)
  const int na = 8 * (m & 1);               // T columns of ta: na .. na + 7; of tb: 16 + na ..
  const int base = (w & 2) ? 32 : 0;        // warps 0..3: (D0, L10, D1) at 0, (D2, L32, D3) at 32
  const int nx = base + 8 * (w & 1);        // X tile columns
  if (w < 4) {
    uint32_t af_[4], bf[2], bt[2];
    float y[4] = {0.f, 0.f, 0.f, 0.f};
    lh_afrag(Lh, base + 16, base, gid, tig, af_);           // L10 / L32
    lh_bfrag(Lh, base, nx, gid, tig, bf);                   // D0 / D2, columns nx ..
    mma_f16_16816(y, af_, bf);
    acc_to_bfrag_h(y, c.lane, bt);
    lh_afrag(Lh, base + 16, base + 16, gid, tig, af_);      // D1 / D3
    mma_f16_16816(x, af_, bt);                              // x = D1 L10 D0 (tile); X = -x
  } else {
    uint32_t af_[4], bf[2];
    lh_afrag(Lh, 32 + tr, 0, gid, tig, af_);                // L21a
    lh_bfrag(Lh, 0, na, gid, tig, bf);                      // D0
    mma_f16_16816(ta, af_, bf);
    lh_afrag(Lh, 32 + tr, 16, gid, tig, af_);               // L21b
    lh_bfrag(Lh, 16, 16 + na, gid, tig, bf);                // D1
    mma_f16_16816(tb, af_, bf);
  }
  tc::named_bar_sync(c.bar, kPrepThreads);                  // L10 and L32 are read
  if (w < 4) {
    const float nxv[4] = {-x[0], -x[1], -x[2], -x[3]};
    lh_store_acc(Lh, base + 16, nx, gid, tig, nxv);
    af_store_neg_acc(af, base + 16, nx, gid, tig, x);
  }
  tc::named_bar_sync(c.bar, kPrepThreads);                  // X10 (and X32) in the scratch
  if (w >= 4) {
    uint32_t af_[4], bf[2];
    lh_afrag(Lh, 32 + tr, 16, gid, tig, af_);               // L21b
    lh_bfrag(Lh, 16, na, gid, tig, bf);                     // X10, columns na ..
    mma_f16_16816(ta, af_, bf);
    lh_store_acc(Lh, tr, 32 + na, gid, tig, ta);            // T -> rows 0..31, columns 32..63
    lh_store_acc(Lh, tr, 48 + na, gid, tig, tb);
  }
  tc::named_bar_sync(c.bar, kPrepThreads);                  // T in the scratch
  {
    const int rb = w >> 2, nt = w & 3;                      // A21 rows 32 + 16 rb .., columns 8 nt ..
    uint32_t af_[4], bf[2];
    float y[4] = {0.f, 0.f, 0.f, 0.f};
    lh_bfrag(Lh, 0, 32 + 8 * nt, gid, tig, bf);             // T_top
    if (rb == 0) {
      lh_afrag(Lh, 32, 32, gid, tig, af_);                  // D2
      mma_f16_16816(y, af_, bf);
    } else {
      lh_afrag(Lh, 48, 32, gid, tig, af_);                  // X32
      mma_f16_16816(y, af_, bf);
      lh_bfrag(Lh, 16, 32 + 8 * nt, gid, tig, bf);          // T_bot
      lh_afrag(Lh, 48, 48, gid, tig, af_);                  // D3
      mma_f16_16816(y, af_, bf);
    }
    af_store_neg_acc(af, 32 + 16 * rb, 8 * nt, gid, tig, y);
  }
}

// A2 = A diag(beta) and B2 = A diag(beta exp(gam)) -> bf16 (128B-swizzled rows at a2_addr,
// b2_addr) from A in fp32 (af, the stored-A layout); thread: 16 columns of one row. kNorm: B2
// multiplies the raw K tile, so its columns also take rk.
template <bool kNorm = false>
__device__ __forceinline__ void prep_store_a_f32(const PrepCtx& c, int s, const float* af, uint32_t a2_addr,
                                                 uint32_t b2_addr) {
  const int i = c.pt & 63, qq = c.pt >> 6;
  const float* bet = c.cs->bet[s];
  const float* ek = kNorm ? c.cs->egk[s] : c.cs->eg[s];
  float a[16];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float4 t = *reinterpret_cast<const float4*>(af + i * kChunk + a_chunk(i, 4 * qq + u) * 4);
    a[4 * u] = t.x; a[4 * u + 1] = t.y; a[4 * u + 2] = t.z; a[4 * u + 3] = t.w;
  }
  uint32_t w2[8], wb[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int j0 = qq * 16 + 2 * u;
    const float b0 = bet[j0], b1 = bet[j0 + 1];
    w2[u] = tc::pack_bf16(a[2 * u] * b0, a[2 * u + 1] * b1);
    wb[u] = tc::pack_bf16(a[2 * u] * (b0 * ek[j0]), a[2 * u + 1] * (b1 * ek[j0 + 1]));
  }
  st_shared_v4(a2_addr + tc::sw128(i, 2 * qq), w2[0], w2[1], w2[2], w2[3]);
  st_shared_v4(a2_addr + tc::sw128(i, 2 * qq + 1), w2[4], w2[5], w2[6], w2[7]);
  st_shared_v4(b2_addr + tc::sw128(i, 2 * qq), wb[0], wb[1], wb[2], wb[3]);
  st_shared_v4(b2_addr + tc::sw128(i, 2 * qq + 1), wb[4], wb[5], wb[6], wb[7]);
}

// A2 = A diag(beta) and A -> bf16 (128B-swizzled rows at a2_addr, a_addr) from the fp32 rows
// of A (stride kLd) in the scratch (thread: 16 columns of one row; a warp covers 32
// consecutive rows of one 16-column quarter).
// (a_addr == 0: A2 only)
__device__ __forceinline__ void prep_write_a_rows(const PrepCtx& c, int s, uint32_t a2_addr, uint32_t a_addr) {
  const int i = c.pt & 63, qq = c.pt >> 6;
  const float* bet = c.cs->bet[s];
  float a[16];
  const float4* src = reinterpret_cast<const float4*>(c.Lf + i * kLd + qq * 16);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float4 t = src[u];
    a[4 * u] = t.x; a[4 * u + 1] = t.y; a[4 * u + 2] = t.z; a[4 * u + 3] = t.w;
  }
  uint32_t w[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int j0 = qq * 16 + 2 * u;
    w[u] = tc::pack_bf16(a[2 * u] * bet[j0], a[2 * u + 1] * bet[j0 + 1]);
  }
  st_shared_v4(a2_addr + tc::sw128(i, 2 * qq), w[0], w[1], w[2], w[3]);
  st_shared_v4(a2_addr + tc::sw128(i, 2 * qq + 1), w[4], w[5], w[6], w[7]);
  if (a_addr) {
#pragma unroll
    for (int u = 0; u < 8; ++u) w[u] = tc::pack_bf16(a[2 * u], a[2 * u + 1]);
    st_shared_v4(a_addr + tc::sw128(i, 2 * qq), w[0], w[1], w[2], w[3]);
    st_shared_v4(a_addr + tc::sw128(i, 2 * qq + 1), w[4], w[5], w[6], w[7]);
  }
}

// Start fetching a chunk's A (fp32 64 x 64 rows in global memory) into the scratch as rows of
// stride kLd, 4 x 16 bytes per thread of a 256-thread group (completion: cp_async_wait_all).
__device__ __forceinline__ void prep_fetch_a(const PrepCtx& c, const float* a_g) {
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int idx = c.pt + kPrepThreads * m, ar = idx >> 4, c16 = idx & 15;
    tc::cp_async_16(tc::smem_u32(c.Lf + ar * kLd + c16 * 4), a_g + ar * kChunk + a_chunk(ar, c16) * 4);
  }
  tc::cp_async_commit();
}

}  // namespace gdn
