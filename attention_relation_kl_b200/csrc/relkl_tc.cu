// tcgen05 / TMA kernels (sm_100a) for the linear-memory relation KL.
//
// LinearARD (arXiv 2604.00004; pith.science verdict, pith_extraction.
// key_machinery) computes, per (batch, head, relation) unit,
//   Z_m = X_m X_m^T * s + M,  R_m = softmax_rows(Z_m),  kl_i = KL(R_t(i,:) || R_s(i,:)),
// keeping only O(N) row statistics (Phase 1) and recomputing the logit tiles
// in the backward pass (Phase 2), where G = dkl (R_s - R_t) and
// dX_s = s (G + G^T) X_s.
//
// Every kernel here is persistent (one CTA per SM, static schedule) and
// warp-specialised:
//   * one TMA warp streams bf16 tiles of X_t and X_s into 128-byte swizzled
//     shared memory (the row blocks of a work item stay resident, column tiles
//     pass through rings);
//   * one or two MMA warps issue tcgen05.mma (kind::f16, M=128) whose fp32
//     accumulators live in tensor memory: the teacher and student logit tiles
//     side by side, and in the backward also the row-side product
//     dX_I += G X_s[J] and the column-side product P = G^T X_s[I] (or its
//     transpose);
//   * four "row" warpgroups read the logit tiles from TMEM (each owns a slice
//     of the tile's columns) and do the per-entry work: the shared-max online
//     softmax and KL sums in the forward, the gradient tile G (bf16, written
//     to shared memory as an MMA operand) in the backward;
//   * in the backward an epilogue warpgroup stages the column-side product and,
//     at the end of a row block, the dX_I accumulator as 32 x 32 fp32 boxes in
//     shared memory and adds them into dX with TMA bulk-tensor reduce-adds
//     (the additions happen in L2).
//
// Work items pair row block p with row block nblk-1-p of the same unit, so
// every causal item holds nblk+1 column tiles and the static round-robin over
// items is balanced; consecutive items belong to the same unit, which keeps
// the unit's X tiles and dX rows resident in L2 while its items run.
//
// Every mbarrier wait is bounded (see relkl_device.cuh): a wait that runs out
// records its site in the caller's workspace, and every role then leaves its
// loop, waits for its own copies and MMAs in flight and the CTA frees its TMEM
// and exits.
#include <cstdint>
#include <cstdio>
#include <vector>
#include <cuda.h>
#include <cuda_runtime.h>

#include "relkl_device.cuh"
#include "relkl_params.h"

namespace relkl {

constexpr int BM = 128;        // rows of a row block (TMEM lanes)
constexpr int BN = 128;        // columns of a logit tile
constexpr int BOX = 128 * 128;  // bytes of one 128-row x 64-col bf16 box
constexpr float kLog2e = 1.4426950408889634f;

constexpr unsigned long long kDrainNs = 200000000ull;  // 0.2 s for in-flight copies

struct Unit {
  const TcSeg* seg;
  int b, h;        // TMA batch and head coordinates
  long long row0;  // first row of the unit in the [B,H,N] arrays (kl, stats, dkl)
  int tok0;        // TMA row coordinate of the unit's first row (packed sequences), else 0
  int len;         // valid rows and columns of the unit
  int span;        // rows the unit's work items cover: len for packed sequences, else N
  int nblk;        // ceil(span / 128)
};

__host__ __device__ constexpr int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int imax(int a, int b) { return a > b ? a : b; }

// Unit u of the launch.  Units of a batched relation are (b, h) of its
// [B, H, N, d] tensors, right-padded to a per-batch length when lengths are
// given; units of packed sequences are (sequence k, head h) of [1, H, N, d]
// tensors holding the sequences back to back, sequence k on tokens
// [cu_seqlens[k], cu_seqlens[k+1]).  `src` reads a segment's lengths and
// sequence offsets (device memory in the kernels, host copies in the
// schedule check).
template <class Src>
__host__ __device__ __forceinline__ Unit make_unit(const TcParams& p, int u, const Src& src) {
  int r = 0;
#pragma unroll
  for (int k = 1; k < kMaxSeg; ++k)
    if (k < p.n_seg && u >= p.seg[k].unit_begin) r = k;
  const TcSeg* s = &p.seg[r];
  const int local = u - s->unit_begin;
  Unit out;
  out.seg = s;
  if (s->cu_seqlens) {
    const int k = local / s->H;
    out.b = 0;
    out.h = local - k * s->H;
    const int a = imin(imax(src.cu(r, k), 0), p.N);
    const int e = imin(imax(src.cu(r, k + 1), a), p.N);
    out.tok0 = a;
    out.len = imin(e - a, s->max_seqlen);
    out.span = out.len;
    out.row0 = static_cast<long long>(out.h) * p.N + a;
  } else {
    out.b = local / s->H;
    out.h = local - out.b * s->H;
    out.tok0 = 0;
    out.len = s->lengths ? imax(0, imin(p.N, src.len(r, out.b))) : p.N;
    out.span = p.N;
    out.row0 = (static_cast<long long>(out.b) * s->H + out.h) * p.N;
  }
  out.nblk = (out.span + BM - 1) / BM;
  return out;
}

struct DeviceUnitSrc {
  const TcParams& p;
  __device__ int len(int r, int b) const { return p.seg[r].lengths[b]; }
  __device__ int cu(int r, int k) const { return p.seg[r].cu_seqlens[k]; }
};

__device__ __forceinline__ Unit decode_unit(const TcParams& p, int u) {
  return make_unit(p, u, DeviceUnitSrc{p});
}

// Work item -> (unit u, per-unit item index pp).  A call that covers one part
// of the work takes the unit's items part, part + n_parts, ...
__host__ __device__ __forceinline__ void decode_item(const TcParams& p, int item, int& u, int& pp) {
  u = item / p.n_local;
  pp = p.part + (item - u * p.n_local) * p.n_parts;
}

// Row blocks of one work item: pass 0 is the longer block nblk-1-p, pass 1
// (absent when both coincide) is block p.  An item index past the unit's
// own pair count (a short packed sequence) has no pass.
__host__ __device__ __forceinline__ int item_passes(const Unit& U, int pp) {
  if (pp >= (U.nblk + 1) / 2) return 0;
  return (pp == U.nblk - 1 - pp) ? 1 : 2;
}
__host__ __device__ __forceinline__ int pass_block(const Unit& U, int pp, int pass) {
  return pass == 0 ? U.nblk - 1 - pp : pp;
}
__host__ __device__ __forceinline__ int n_col_tiles(const TcParams& p, const Unit& U, int I) {
  return p.causal ? I + 1 : U.nblk;
}

// Issue the K-loop of one M=128 x N=128 logit tile: acc = A_tile * B_tile^T
// with both operands K-major (rows of X, d contiguous), K = D.
template <int D>
__device__ __forceinline__ void issue_logits(uint32_t acc, uint32_t a_base, uint32_t b_base) {
  constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
#pragma unroll
  for (int k = 0; k < D / 16; ++k) {
    const uint32_t off = (k >> 2) * BOX + (k & 3) * 32;
    umma_bf16(acc, sw128_desc(a_base + off, 16, 1024), sw128_desc(b_base + off, 16, 1024), idesc,
              k > 0 ? 1u : 0u);
  }
}

// Same K-loop with precomputed descriptor words: a_lo and b_lo name the first
// 64-column box of 128-row tiles (boxes 16 KB apart), steps of 32 B in a row.
template <int D>
__device__ __forceinline__ void issue_logits_w(uint32_t lead, uint32_t acc, uint32_t a_lo,
                                               uint32_t b_lo) {
  constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
  constexpr uint32_t hi = sw128_desc_hi(1024);
#pragma unroll
  for (int k = 0; k < D / 16; ++k) {
    const uint32_t off = (k >> 2) * (BOX >> 4) + (k & 3) * 2;
    umma_bf16_w_lead(lead, acc, a_lo + off, hi, b_lo + off, hi, idesc, k > 0 ? 1u : 0u);
  }
}

// =========================================================================
//                                FORWARD
// =========================================================================
template <int D>
struct FwdSmem {
  static constexpr int TILE = BM * D * 2;
  static constexpr int XT_I = 0;
  static constexpr int XS_I = TILE;
  static constexpr int RING = 2 * TILE;              // stage k: xt at RING + 2k*TILE, xs after it
  static constexpr int STAGES = 2;
  static constexpr int MERGE = RING + STAGES * 2 * TILE;  // float4 per row, 3 column quarters
  static constexpr int BARS = MERGE + 3 * BM * 16;
  // barriers: full_I, empty_I, full_J[2], empty_J[2], tf[2], te[2], mfull, mempty, drain
  static constexpr int NBAR = 13;
  static constexpr int MISC = BARS + NBAR * 8;       // tmem base (u32) + abort flag (int)
  static constexpr int BYTES = MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;         // slack for 1024-byte alignment
};

// Warps 0-15: four row warpgroups, warpgroup k owning columns [32k, 32k+32)
// of every tile; warp 16 TMA; warp 17 MMA.
constexpr int FWD_THREADS = 576;
constexpr int FWD_TMA_WARP = 16, FWD_MMA_WARP = 17;

template <int D>
__global__ void __launch_bounds__(FWD_THREADS, 1)
relkl_fwd_tc_kernel(const __grid_constant__ TcParams p) {
  using L = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t bar0 = base + L::BARS;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * i; };
  const uint32_t FULL_I = BAR(0), EMPTY_I = BAR(1);
  auto FULL_J = [&](int s) { return BAR(2 + s); };
  auto EMPTY_J = [&](int s) { return BAR(4 + s); };
  auto TF = [&](int b) { return BAR(6 + b); };
  auto TE = [&](int b) { return BAR(8 + b); };
  const uint32_t MFULL = BAR(10), MEMPTY = BAR(11), DRAIN = BAR(12);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::MISC + 4);
  float4* merge = reinterpret_cast<float4*>(gbase + L::MERGE);

  WaitCtl wc{p.status, abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(FULL_I, 1);
    mbar_init(EMPTY_I, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(FULL_J(s), 1);
      mbar_init(EMPTY_J(s), 1);
      mbar_init(TF(s), 1);
      mbar_init(TE(s), 16);
    }
    mbar_init(MFULL, 12);
    mbar_init(MEMPTY, 4);
    mbar_init(DRAIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == FWD_MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == FWD_TMA_WARP) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      for (int s = 0; s < p.n_seg; ++s) {
        tma_prefetch_desc(&p.seg[s].tm_t);
        tma_prefetch_desc(&p.seg[s].tm_s);
      }
      uint32_t nI = 0, nJ = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        int u, pp;
        decode_item(p, item, u, pp);
        const Unit U = decode_unit(p, u);
        for (int pass = 0; ok && pass < item_passes(U, pp); ++pass) {
          const int I = pass_block(U, pp, pass);
          if (!(ok = mbar_wait(EMPTY_I, (nI & 1) ^ 1, wc, W_TMA_EMPTY_I))) break;
          mbar_arrive_expect_tx(FULL_I, 2 * L::TILE);
#pragma unroll
          for (int b = 0; b < D / 64; ++b) {
            tma_load_4d(base + L::XT_I + b * BOX, &U.seg->tm_t, FULL_I, b * 64, U.tok0 + I * BM, U.h, U.b);
            tma_load_4d(base + L::XS_I + b * BOX, &U.seg->tm_s, FULL_I, b * 64, U.tok0 + I * BM, U.h, U.b);
          }
          ++nI;
          const int nT = n_col_tiles(p, U, I);
          for (int J = 0; J < nT; ++J) {
            const int st = nJ & 1;
            if (!(ok = mbar_wait(EMPTY_J(st), ((nJ >> 1) & 1) ^ 1, wc, W_TMA_EMPTY_J))) break;
            const uint32_t xt = base + L::RING + st * 2 * L::TILE;
            mbar_arrive_expect_tx(FULL_J(st), 2 * L::TILE);
#pragma unroll
            for (int b = 0; b < D / 64; ++b) {
              tma_load_4d(xt + b * BOX, &U.seg->tm_t, FULL_J(st), b * 64, U.tok0 + J * BN, U.h, U.b);
              tma_load_4d(xt + L::TILE + b * BOX, &U.seg->tm_s, FULL_J(st), b * 64, U.tok0 + J * BN,
                          U.h, U.b);
            }
            ++nJ;
          }
        }
      }
      // wait for the copies still in flight before the CTA may exit
      if (nI) mbar_wait_drain(FULL_I, (nI - 1) & 1, kDrainNs);
      for (int st = 0; st < 2; ++st) {
        const uint32_t arms = (nJ + 1 - st) / 2;
        if (arms) mbar_wait_drain(FULL_J(st), (arms - 1) & 1, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp == FWD_MMA_WARP) {
    // ------------------------------------------------------------ MMA
    // The whole warp runs this loop (descriptor words stay warp-uniform); one
    // elected lane issues the MMAs and commits.
    {
      const uint32_t lead = elect_leader();
      uint32_t nI = 0, nJ = 0, nt = 0;
      bool ok = true, issued = false;
      const uint32_t dXtI = sw128_desc_lo(base + L::XT_I, 16);
      const uint32_t dXsI = sw128_desc_lo(base + L::XS_I, 16);
      const uint32_t ring0 = sw128_desc_lo(base + L::RING, 16);
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        int u, pp;
        decode_item(p, item, u, pp);
        const Unit U = decode_unit(p, u);
        for (int pass = 0; ok && pass < item_passes(U, pp); ++pass) {
          const int I = pass_block(U, pp, pass);
          if (!(ok = mbar_wait_warp(FULL_I, nI & 1, wc, W_MMA_FULL_I))) break;
          const int nT = n_col_tiles(p, U, I);
          for (int J = 0; J < nT; ++J) {
            const int st = nJ & 1;
            const int buf = nt & 1;
            if (!(ok = mbar_wait_warp(FULL_J(st), (nJ >> 1) & 1, wc, W_MMA_FULL_J))) break;
            if (!(ok = mbar_wait_warp(TE(buf), ((nt >> 1) & 1) ^ 1, wc, W_MMA_S_EMPTY))) break;
            tc_fence_after();
            const uint32_t xt = ring0 + st * (2 * L::TILE >> 4);
            const uint32_t acc = tmem + buf * 256;
            issue_logits_w<D>(lead, acc, dXtI, xt);
            issue_logits_w<D>(lead, acc + 128, dXsI, xt + (L::TILE >> 4));
            issued = true;
            umma_commit_lead(lead, EMPTY_J(st));
            umma_commit_lead(lead, TF(buf));
            ++nJ;
            ++nt;
          }
          if (!ok) break;
          umma_commit_lead(lead, EMPTY_I);
          ++nI;
        }
      }
      if (issued) {
        umma_commit_lead(lead, DRAIN);
        mbar_wait_drain(DRAIN, 0, kDrainNs);
      }
    }
    __syncwarp();
  } else {
    // --------------------------------------------------- row warpgroups
    static_assert(2 * 2 * BN <= 512, "TMEM columns: 2 x (Z_t, Z_s)");
    const int q = warp & 3;      // TMEM lane quarter
    const int wg = warp >> 2;    // column quarter of each tile
    const int r = q * 32 + lane;
    const float sl2 = p.sl2;
    uint32_t nt = 0, nm = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      int u, pp;
        decode_item(p, item, u, pp);
      const Unit U = decode_unit(p, u);
      for (int pass = 0; ok && pass < item_passes(U, pp); ++pass) {
        const int I = pass_block(U, pp, pass);
        const int row = I * BM + r;
        const int nT = n_col_tiles(p, U, I);
        const int L = U.len;
        float m_run = -INFINITY;
        // running sums, two float2 lanes each: S_t, C = sum(e_s - e_t), A = sum e_t (z_t - z_s)
        float2 S2[2], C2[2], A2[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) S2[k] = C2[k] = A2[k] = make_float2(0.f, 0.f);
        for (int J = 0; J < nT; ++J) {
          const int buf = nt & 1;
          ok = mbar_wait(TF(buf), (nt >> 1) & 1, wc, W_SM_S_FULL);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * 256 + wg * 32;
          float t[32], s[32];
          tmem_ld32(ta, t);
          tmem_ld32(ta + 128, s);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(TE(buf));
          ++nt;
          const int col0 = J * BN + wg * 32;
          const bool need_mask = (p.causal && J == I) || (col0 + 32 > L);
          if (!need_mask) {
            float m4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) m4[k] = fmaxf(t[k], s[k]);
#pragma unroll
            for (int k = 4; k < 32; ++k) m4[k & 3] = fmaxf(m4[k & 3], fmaxf(t[k], s[k]));
            const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            if (mx > m_run) {
              const float a = ex2_approx((m_run - mx) * sl2);
              const float2 a2 = make_float2(a, a);
#pragma unroll
              for (int k = 0; k < 2; ++k) {
                S2[k] = __fmul2_rn(S2[k], a2);
                C2[k] = __fmul2_rn(C2[k], a2);
                A2[k] = __fmul2_rn(A2[k], a2);
              }
              m_run = mx;
            }
            const float nb = -m_run * sl2;
            const float2 sl2v = make_float2(sl2, sl2), nbv = make_float2(nb, nb);
            const float2 m1 = make_float2(-1.f, -1.f);
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
              const float2 tv = make_float2(t[k], t[k + 1]);
              const float2 sv = make_float2(s[k], s[k + 1]);
              const float2 at = __ffma2_rn(tv, sl2v, nbv);
              const float2 as = __ffma2_rn(sv, sl2v, nbv);
              const float2 et = ex2_approx2(at), es = ex2_approx2(as);
              const int a = (k >> 1) & 1;
              S2[a] = __fadd2_rn(S2[a], et);
              C2[a] = __fadd2_rn(C2[a], __ffma2_rn(et, m1, es));
              A2[a] = __ffma2_rn(et, __ffma2_rn(sv, m1, tv), A2[a]);
            }
          } else {
            // diagonal or ragged tile: per-entry predicate
            const int lim = row >= L ? -1 : (p.causal ? min(row, L - 1) : L - 1);
            float mx = -INFINITY;
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (col0 + k <= lim) mx = fmaxf(mx, fmaxf(t[k], s[k]));
            if (mx > m_run) {
              const float a = ex2_approx((m_run - mx) * sl2);
              const float2 a2 = make_float2(a, a);
#pragma unroll
              for (int k = 0; k < 2; ++k) {
                S2[k] = __fmul2_rn(S2[k], a2);
                C2[k] = __fmul2_rn(C2[k], a2);
                A2[k] = __fmul2_rn(A2[k], a2);
              }
              m_run = mx;
            }
            if (m_run > -INFINITY) {
              const float nb = -m_run * sl2;
#pragma unroll
              for (int k = 0; k < 32; ++k) {
                if (col0 + k <= lim) {
                  const float et = ex2_approx(fmaf(t[k], sl2, nb));
                  const float es = ex2_approx(fmaf(s[k], sl2, nb));
                  float2& Sa = S2[(k >> 1) & 1];
                  float2& Ca = C2[(k >> 1) & 1];
                  float2& Aa = A2[(k >> 1) & 1];
                  if (k & 1) {
                    Sa.y += et;
                    Ca.y += es - et;
                    Aa.y = fmaf(et, t[k] - s[k], Aa.y);
                  } else {
                    Sa.x += et;
                    Ca.x += es - et;
                    Aa.x = fmaf(et, t[k] - s[k], Aa.x);
                  }
                }
              }
            }
          }
        }
        if (!ok) break;
        const float Sx = (S2[0].x + S2[0].y) + (S2[1].x + S2[1].y);
        const float Cx = (C2[0].x + C2[0].y) + (C2[1].x + C2[1].y);
        const float Ax = (A2[0].x + A2[0].y) + (A2[1].x + A2[1].y);
        // merge the four column quarters through shared memory
        if (wg != 0) {
          ok = mbar_wait(MEMPTY, (nm & 1) ^ 1, wc, W_SM_S_FULL);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          merge[(wg - 1) * BM + r] = make_float4(m_run, Sx, Cx, Ax);
          __syncwarp();
          if (lane == 0) mbar_arrive(MFULL);
        } else {
          ok = mbar_wait(MFULL, nm & 1, wc, W_SM_S_FULL);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          const float4 o1 = merge[r], o2 = merge[BM + r], o3 = merge[2 * BM + r];
          __syncwarp();
          if (lane == 0) mbar_arrive(MEMPTY);
          const float M = fmaxf(fmaxf(m_run, o1.x), fmaxf(o2.x, o3.x));
          const float a0 = ex2_approx((m_run - M) * sl2);
          const float a1 = ex2_approx((o1.x - M) * sl2);
          const float a2 = ex2_approx((o2.x - M) * sl2);
          const float a3 = ex2_approx((o3.x - M) * sl2);
          const float St = (Sx * a0 + o1.y * a1) + (o2.y * a2 + o3.y * a3);
          const float Ct = (Cx * a0 + o1.z * a1) + (o2.z * a2 + o3.z * a3);
          const float At = (Ax * a0 + o1.w * a1) + (o2.w * a2 + o3.w * a3);
          const long long g = U.row0 + row;
          if (row < L) {
            const float mz = M * p.scale;
            const float lse_t = mz + logf(St);
            const float rc = Ct / St;
            const float l1 = log1pf(rc);
            const float w = p.scale * At / St;
            U.seg->kl[g] = w + l1;
            reinterpret_cast<float4*>(U.seg->stats)[g] = make_float4(mz, lse_t, lse_t + l1, w);
          } else if (row < U.span) {   // padding row (a packed sequence has none: span = len)
            U.seg->kl[g] = 0.f;
            reinterpret_cast<float4*>(U.seg->stats)[g] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        ++nm;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == FWD_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =========================================================================
//                                BACKWARD
// =========================================================================
// Phase 2 on the pages: recompute the logit tiles, rebuild R_t and R_s from
// the stored LSEs, form G = dkl (R_s - R_t) (bf16, in shared memory) and
// stream it into dX_s = s (G X_s[J] for the row block, G^T X_s[I] for the
// column block).  Three kernels share the work: one 128-row block per pass
// (d = 128, causal, few row blocks), adjacent row-block pairs (d = 128
// otherwise) and adjacent pairs with 128-column tiles (d = 64).
// Warps 0-15: four row warpgroups; warps 16-19: epilogue; warp 20: TMA;
// warp 21 (and 22 in the paired kernels): MMA.
constexpr int BWD_THREADS = 704;
constexpr int BWD_EPI_WARP = 16, BWD_TMA_WARP = 20, BWD_MMA_WARP = 21;

// Epilogue helper: add the 32 rows x D columns a warp holds in TMEM
// (lanes q*32.., columns col0..) into dX rows row0.. through TMA reduce-adds
// of 32 x 32 f32 boxes staged in 128B-swizzled shared memory (two buffers per
// warp).  Rows at or past N are skipped by TMA.
template <int D>
__device__ __forceinline__ void epilogue_reduce(uint32_t taddr, uint32_t stg, uint32_t& nstg,
                                                const CUtensorMap* map, int row0, int h, int b,
                                                int N, int lane, uint32_t release_bar) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    tmem_wait_ld();
    if (c == D / 32 - 1) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(release_bar);
    }
    const uint32_t buf = stg + (nstg & 1) * (32 * 32 * 4);
    if (lane == 0) bulk_wait_read<1>();   // this buffer's previous reduce has read it
    __syncwarp();
    const uint32_t rowp = buf + lane * 128;
#pragma unroll
    for (int k4 = 0; k4 < 8; ++k4)
      st_shared_v4(rowp + ((k4 ^ (lane & 7)) << 4), __float_as_uint(v[4 * k4]),
                   __float_as_uint(v[4 * k4 + 1]), __float_as_uint(v[4 * k4 + 2]),
                   __float_as_uint(v[4 * k4 + 3]));
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (row0 < N) tma_reduce_add_4d(map, buf, c * 32, row0, h, b);
      bulk_commit();
    }
    ++nstg;
  }
}

// =========================================================================
//              BACKWARD, d = 128: 64-column tiles, double-buffered
// =========================================================================
// One 128-row block per pass with column tiles of 64: the logit
// tiles (2 x 64 TMEM columns), the gradient tile G (16 KB) and the transposed
// column-side product P^T = X_s[I]^T G (64 TMEM columns, M = d = 128) are all
// double-buffered, and the student column tiles pass through a 4-stage ring, so
// that the exp pass of tile t overlaps the logit MMAs of tile t+1 and the
// gradient MMAs of tile t-1 without waiting on a shared buffer.
//   TMEM: Z_t/Z_s buffers 0..255 (128 per buffer), dX_I 256..383, P^T 384..511.
//   smem: X_t[I], X_s[I] 32 KB each; teacher ring 2 x 16 KB; student ring
//         4 x 16 KB; G 2 x 16 KB; epilogue staging 32 KB.
struct Bwd64Smem {
  static constexpr int TILE_I = BM * 128 * 2;        // 128 rows: boxes of 128 x 64 (16 KB)
  static constexpr int TILE_J = 64 * 128 * 2;        // 64 rows: boxes of 64 x 64 (8 KB)
  static constexpr int BOX_J = 64 * 128;
  static constexpr int XT_I = 0;
  static constexpr int XS_I = TILE_I;
  static constexpr int XT_R = 2 * TILE_I;            // 2 stages
  static constexpr int XS_R = XT_R + 2 * TILE_J;     // 4 stages
  static constexpr int G = XS_R + 4 * TILE_J;        // 2 x (128 x 64 bf16)
  static constexpr int G_BYTES = BM * 64 * 2;
  static constexpr int STG = G + 2 * G_BYTES;
  static constexpr int STG_BYTES = 32 * 32 * 4;
  static constexpr int BARS = STG + 4 * 2 * STG_BYTES;
  // full_I, empty_I, fullT[2], emptyT[2], fullS[4], emptyS[4], s_full[2], s_empty[2],
  // g_full[2], (2 spare), p_full[2], p_empty[2], dxi_full, dxi_empty, drain
  static constexpr int NBAR = 31;
  static constexpr int MISC = BARS + NBAR * 8;
  static constexpr int BYTES = MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
};
static_assert(Bwd64Smem::ALLOC <= 232448, "backward shared memory exceeds 227 KB");

constexpr int BN64 = 64;

// Column tiles of row block I in the paired-block kernels.  With SYM (full
// masks) only the tiles up to the diagonal block are visited, as under the
// causal mask: each off-diagonal tile then serves both orientations of its
// entries (Z = Z^T).
template <bool SYM>
__host__ __device__ __forceinline__ int n_col_tiles64_s(const TcParams& p, const Unit& U, int I) {
  const int nb64 = (U.span + BN64 - 1) / BN64;
  return (p.causal || SYM) ? imin(2 * I + 2, nb64) : nb64;
}
template <bool SYM>
__host__ __device__ __forceinline__ int n_col_tiles_s(const TcParams& p, const Unit& U, int I) {
  return (p.causal || SYM) ? I + 1 : U.nblk;
}

// Row-side G plus, for an entry (i, j) off the diagonal block of a full mask,
// its transposed partner G(j, i) = dkl_j (R_s - R_t)(j, i), which reuses the
// logits because Z(j, i) = Z(i, j).  Row j's LSEs and upstream gradient come
// from the statistics of column j: before the tile's logits arrive, lane l of
// each warp loads the constants of one of the warp's columns
// (partner_column), and the entries take them from that lane by shuffles.
struct PartnerCol {
  float bt, bs, mul;   // -lse_t log2 e, -lse_s log2 e, dkl * scale of one column
  float ut, us;        // mul * 2^(bt - c_t), mul * 2^(bs - c_s): the column's share of the rescale
};

__device__ __forceinline__ PartnerCol partner_column(const Unit& U, const TcParams& p, int c) {
  const int cc = imin(c, U.span - 1);   // columns past the unit are masked; keep the load inside
  const float4 a = reinterpret_cast<const float4*>(U.seg->stats)[U.row0 + cc];
  PartnerCol out;
  out.bt = -a.y * kLog2e;
  out.bs = -a.z * kLog2e;
  out.mul = (U.seg->dkl ? U.seg->dkl[U.row0 + cc] : 1.0f / static_cast<float>(U.len)) * p.scale;
  out.ut = out.us = 0.f;
  return out;
}

// The partner of entry (i, j) is dkl_j (2^(zs l + bs_j) - 2^(zt l + bt_j)) with
// l = scale log2 e.  Since 2^(zs l + bs_j) = 2^(zs l + bs_i) 2^(bs_j - bs_i), it
// reuses the row side's exps: with a per-tile reference c (the first column's
// bs), 2^(bs_j - bs_i) = 2^(c - bs_i) 2^(bs_j - c), a per-row times a
// per-column factor, so H(i,j) = es (m_i + A_i^s u_j^s) - et (m_i + A_i^t u_j^t)
// costs 2 exps per entry instead of 4.  Valid while every factor stays well
// inside float range: |bs - c| <= 43 for the rows and columns of the tile (the
// LSEs then differ by at most ~60, and a partner whose row-side exp
// underflows is below 2^-80 of its column's largest term); a warp whose tile
// leaves that range takes the 4-exp form.
struct PartnerTile {
  float at, as;   // 2^(c_t - bt_i), 2^(c_s - bs_i) of this thread's row
  bool ok;        // the factored form holds for this warp's tile
};

__device__ __forceinline__ PartnerTile partner_tile(PartnerCol& pc, float bt_i, float bs_i) {
  constexpr unsigned kAll = 0xffffffffu;
  const float ct = __shfl_sync(kAll, pc.bt, 0), cs = __shfl_sync(kAll, pc.bs, 0);
  const bool in = fabsf(ct - bt_i) <= 43.f && fabsf(cs - bs_i) <= 43.f &&
                  fabsf(pc.bt - ct) <= 43.f && fabsf(pc.bs - cs) <= 43.f;
  PartnerTile pt;
  pt.ok = __all_sync(kAll, in);
  pt.at = ex2_approx(ct - bt_i);
  pt.as = ex2_approx(cs - bs_i);
  pc.ut = pc.mul * ex2_approx(pc.bt - ct);
  pc.us = pc.mul * ex2_approx(pc.bs - cs);
  return pt;
}

// Adds the partners of the column pair held by lanes src, src + 1 to g (the
// 4-exp form); zt2 / zs2 are the raw logit accumulators of the pair.
__device__ __forceinline__ float2 sym_partner(const PartnerCol& pc, int src, float sl2, float2 zt2,
                                              float2 zs2, float2 g) {
  constexpr unsigned kAll = 0xffffffffu;
  const float2 btc = make_float2(__shfl_sync(kAll, pc.bt, src), __shfl_sync(kAll, pc.bt, src + 1));
  const float2 bsc = make_float2(__shfl_sync(kAll, pc.bs, src), __shfl_sync(kAll, pc.bs, src + 1));
  const float2 mulc =
      make_float2(__shfl_sync(kAll, pc.mul, src), __shfl_sync(kAll, pc.mul, src + 1));
  const float2 sl2v = make_float2(sl2, sl2);
  const float2 et = ex2_approx2(__ffma2_rn(zt2, sl2v, btc));
  const float2 es = ex2_approx2(__ffma2_rn(zs2, sl2v, bsc));
  return __ffma2_rn(__ffma2_rn(et, make_float2(-1.f, -1.f), es), mulc, g);
}

// The same entries packed into NC/2 bf16 pairs in registers (for callers
// that must wait for the G buffer after forming them).
template <int NC>
__device__ __forceinline__ void form_g_pack(const float (&t)[NC], const float (&s)[NC], float bt,
                                            float bs, float mul, int col0, int lim, bool off,
                                            const PartnerCol& pc, const PartnerTile& pt, int lane0,
                                            const TcParams& p, uint32_t (&pk)[NC / 2]) {
  constexpr unsigned kAll = 0xffffffffu;
  const float2 sl2v = make_float2(p.sl2, p.sl2), btv = make_float2(bt, bt),
               bsv = make_float2(bs, bs), mulv = make_float2(mul, mul),
               m1 = make_float2(-1.f, -1.f), atv = make_float2(pt.at, pt.at),
               asv = make_float2(pt.as, pt.as);
  const bool need_mask = col0 + NC - 1 > lim;
  const bool fac = off && pt.ok;
#pragma unroll
  for (int k = 0; k < NC; k += 2) {
    const float2 zt2 = make_float2(t[k], t[k + 1]), zs2 = make_float2(s[k], s[k + 1]);
    const float2 et = ex2_approx2(__ffma2_rn(zt2, sl2v, btv));
    const float2 es = ex2_approx2(__ffma2_rn(zs2, sl2v, bsv));
    float2 g;
    if (fac) {
      const int src = lane0 + k;
      const float2 ut = make_float2(__shfl_sync(kAll, pc.ut, src), __shfl_sync(kAll, pc.ut, src + 1));
      const float2 us = make_float2(__shfl_sync(kAll, pc.us, src), __shfl_sync(kAll, pc.us, src + 1));
      const float2 ft = __ffma2_rn(atv, ut, mulv), fs = __ffma2_rn(asv, us, mulv);
      g = __ffma2_rn(es, fs, __fmul2_rn(__fmul2_rn(et, ft), m1));
    } else {
      g = __fmul2_rn(__ffma2_rn(et, m1, es), mulv);
      if (off) g = sym_partner(pc, lane0 + k, p.sl2, zt2, zs2, g);
    }
    if (need_mask) {
      g.x = (col0 + k <= lim) ? g.x : 0.f;
      g.y = (col0 + k + 1 <= lim) ? g.y : 0.f;
    }
    pk[k >> 1] = pack_bf16x2(g.x, g.y);
  }
}

template <int NC>
__device__ __forceinline__ void form_g_store(const float (&t)[NC], const float (&s)[NC],
                                             float bt, float bs, float mul, int col0, int lim,
                                             bool off, const PartnerCol& pc, int lane0,
                                             const TcParams& p, uint32_t row_addr, int chunk0,
                                             int r) {
  const float2 sl2v = make_float2(p.sl2, p.sl2), btv = make_float2(bt, bt),
               bsv = make_float2(bs, bs), mulv = make_float2(mul, mul),
               m1 = make_float2(-1.f, -1.f);
  const bool need_mask = col0 + NC - 1 > lim;
#pragma unroll
  for (int q = 0; q < NC / 8; ++q) {
    uint32_t pk[4];
#pragma unroll
    for (int k2 = 0; k2 < 8; k2 += 2) {
      const int k = q * 8 + k2;
      const float2 zt2 = make_float2(t[k], t[k + 1]), zs2 = make_float2(s[k], s[k + 1]);
      const float2 et = ex2_approx2(__ffma2_rn(zt2, sl2v, btv));
      const float2 es = ex2_approx2(__ffma2_rn(zs2, sl2v, bsv));
      float2 g = __fmul2_rn(__ffma2_rn(et, m1, es), mulv);
      if (off) g = sym_partner(pc, lane0 + k, p.sl2, zt2, zs2, g);
      if (need_mask) {
        g.x = (col0 + k <= lim) ? g.x : 0.f;
        g.y = (col0 + k + 1 <= lim) ? g.y : 0.f;
      }
      pk[k2 >> 1] = pack_bf16x2(g.x, g.y);
    }
    st_shared_v4(row_addr + (((chunk0 + q) ^ (r & 7)) << 4), pk[0], pk[1], pk[2], pk[3]);
  }
}

__host__ __device__ __forceinline__ int n_col_tiles64(const TcParams& p, const Unit& U, int I) {
  const int nb64 = (U.span + BN64 - 1) / BN64;
  return p.causal ? imin(2 * I + 2, nb64) : nb64;
}

__global__ void __launch_bounds__(BWD_THREADS, 1)
relkl_bwd_tc64_kernel(const __grid_constant__ TcParams p) {
  using L = Bwd64Smem;
  constexpr int D = 128;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t bar0 = base + L::BARS;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * i; };
  const uint32_t FULL_I = BAR(0), EMPTY_I = BAR(1);
  auto FULL_T = [&](int s) { return BAR(2 + s); };
  auto EMPTY_T = [&](int s) { return BAR(4 + s); };
  auto FULL_S = [&](int s) { return BAR(6 + s); };
  auto EMPTY_S = [&](int s) { return BAR(10 + s); };
  auto S_FULL = [&](int b) { return BAR(14 + b); };
  auto S_EMPTY = [&](int b) { return BAR(16 + b); };
  auto G_FULL = [&](int b) { return BAR(18 + b); };
  auto P_FULL = [&](int b) { return BAR(22 + b); };
  auto P_EMPTY = [&](int b) { return BAR(24 + b); };
  const uint32_t DXI_FULL = BAR(26), DXI_EMPTY = BAR(27), DRAIN = BAR(28);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::MISC + 4);

  WaitCtl wc{p.status, abort_flag, p.timeout_ns};
  constexpr uint32_t T_S = 0, T_DXI = 256, T_P = 384;
  static_assert(T_S + 2 * 2 * BN64 <= T_DXI && T_DXI + D <= T_P && T_P + 2 * BN64 <= 512,
                "TMEM columns: 2 x (Z_t, Z_s) | dX_I | 2 x P^T");

  if (threadIdx.x == 0) {
    mbar_init(FULL_I, 1);
    mbar_init(EMPTY_I, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(FULL_T(s), 1);
      mbar_init(EMPTY_T(s), 1);
      mbar_init(S_FULL(s), 1);
      mbar_init(S_EMPTY(s), 16);
      mbar_init(G_FULL(s), 16);
      mbar_init(P_FULL(s), 1);
      mbar_init(P_EMPTY(s), 4);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(FULL_S(s), 1);
      mbar_init(EMPTY_S(s), 1);
    }
    mbar_init(DXI_FULL, 1);
    mbar_init(DXI_EMPTY, 4);
    mbar_init(DRAIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == BWD_MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == BWD_TMA_WARP) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      for (int s = 0; s < p.n_seg; ++s) {
        tma_prefetch_desc(&p.seg[s].tm_t);
        tma_prefetch_desc(&p.seg[s].tm_s);
        tma_prefetch_desc(&p.seg[s].tm_t64);
        tma_prefetch_desc(&p.seg[s].tm_s64);
        tma_prefetch_desc(&p.seg[s].tm_dx);
      }
      uint32_t nI = 0, nJ = 0;
      uint32_t armsT[2] = {0, 0}, armsS[4] = {0, 0, 0, 0};
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        int u, pp;
        decode_item(p, item, u, pp);
        const Unit U = decode_unit(p, u);
        for (int pass = 0; ok && pass < item_passes(U, pp); ++pass) {
          const int I = pass_block(U, pp, pass);
          if (!(ok = mbar_wait(EMPTY_I, (nI & 1) ^ 1, wc, W_TMA_EMPTY_I))) break;
          mbar_arrive_expect_tx(FULL_I, 2 * L::TILE_I);
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            tma_load_4d(base + L::XT_I + b * BOX, &U.seg->tm_t, FULL_I, b * 64, U.tok0 + I * BM, U.h, U.b);
            tma_load_4d(base + L::XS_I + b * BOX, &U.seg->tm_s, FULL_I, b * 64, U.tok0 + I * BM, U.h, U.b);
          }
          ++nI;
          const int nT = n_col_tiles64(p, U, I);
          for (int J = 0; J < nT; ++J) {
            const int tt = nJ & 1, ts = nJ & 3;
            if (!(ok = mbar_wait(EMPTY_T(tt), ((nJ >> 1) & 1) ^ 1, wc, W_TMA_EMPTY_J))) break;
            mbar_arrive_expect_tx(FULL_T(tt), L::TILE_J);
#pragma unroll
            for (int b = 0; b < 2; ++b)
              tma_load_4d(base + L::XT_R + tt * L::TILE_J + b * L::BOX_J, &U.seg->tm_t64,
                          FULL_T(tt), b * 64, U.tok0 + J * BN64, U.h, U.b);
            ++armsT[tt];
            if (!(ok = mbar_wait(EMPTY_S(ts), ((nJ >> 2) & 1) ^ 1, wc, W_TMA_EMPTY_J))) break;
            mbar_arrive_expect_tx(FULL_S(ts), L::TILE_J);
#pragma unroll
            for (int b = 0; b < 2; ++b)
              tma_load_4d(base + L::XS_R + ts * L::TILE_J + b * L::BOX_J, &U.seg->tm_s64,
                          FULL_S(ts), b * 64, U.tok0 + J * BN64, U.h, U.b);
            ++armsS[ts];
            ++nJ;
          }
        }
      }
      if (nI) mbar_wait_drain(FULL_I, (nI - 1) & 1, kDrainNs);
      for (int s = 0; s < 2; ++s)
        if (armsT[s]) mbar_wait_drain(FULL_T(s), (armsT[s] - 1) & 1, kDrainNs);
      for (int s = 0; s < 4; ++s)
        if (armsS[s]) mbar_wait_drain(FULL_S(s), (armsS[s] - 1) & 1, kDrainNs);
    }
    __syncwarp();
  } else if (warp == BWD_MMA_WARP) {
    // ------------------------------------------------------------ MMA
    // The whole warp runs this loop (descriptor words stay warp-uniform); one
    // elected lane issues the MMAs and commits.
    {
      const uint32_t lead = elect_leader();
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN64, 0, 0);
      constexpr uint32_t IDESC_GX = idesc_bf16_f32(BM, D, 0, 1);    // A = G (K-major), B = X_s[J] (MN)
      constexpr uint32_t IDESC_PT = idesc_bf16_f32(D, BN64, 1, 1);  // A = X_s[I]^T (MN), B = G (MN)
      uint32_t nI = 0, nJ = 0, ns = 0, ng = 0, nrb = 0;
      bool ok = true, issued = false;
      // Low descriptor words of every operand buffer (all share the high word
      // of an 8-row-group stride of 1024 B).  K-major operands step along K by
      // 32 B inside a 128 B row and by one box across 64-column boxes; MN-major
      // operands step by 2 KB (16 rows) and name the next 64-column box in LBO.
      // (a buffer's word is the stage-0 word plus stage * size/16)
      const uint32_t HI_1024 = sw128_desc_hi(1024);
      const uint32_t dXtI_k = sw128_desc_lo(base + L::XT_I, 16);
      const uint32_t dXsI_k = sw128_desc_lo(base + L::XS_I, 16);
      const uint32_t dXsI_mn = sw128_desc_lo(base + L::XS_I, BOX);
      const uint32_t dXtJ_k0 = sw128_desc_lo(base + L::XT_R, 16);
      const uint32_t dXsJ_k0 = sw128_desc_lo(base + L::XS_R, 16);
      const uint32_t dXsJ_mn0 = sw128_desc_lo(base + L::XS_R, L::BOX_J);
      const uint32_t dG_k0 = sw128_desc_lo(base + L::G, 16);
      const uint32_t dG_mn0 = sw128_desc_lo(base + L::G, BOX);
      constexpr uint32_t J_STEP = L::TILE_J >> 4, G_STEP = L::G_BYTES >> 4;
      // gradient MMAs of the tile whose student slot is `ts`; `first` starts dX_I
      auto grad = [&](int ts, bool first) -> bool {
        const int b = ng & 1;
        const uint32_t par = (ng >> 1) & 1;
        if (!mbar_wait_warp(G_FULL(b), par, wc, W_MMA_G_FULL)) return false;
        if (!mbar_wait_warp(P_EMPTY(b), par ^ 1, wc, W_MMA_P_EMPTY)) return false;
        if (first && !mbar_wait_warp(DXI_EMPTY, (nrb & 1) ^ 1, wc, W_MMA_DXI_EMPTY)) return false;
        tc_fence_after();
        const uint32_t g_k = dG_k0 + b * G_STEP, g_mn = dG_mn0 + b * G_STEP;
        const uint32_t xsj = dXsJ_mn0 + ts * J_STEP;
        // dX_I += G X_s[J]: M = i, N = c, K = j (64); K steps of 32 B (G) and 2 KB (X_s[J])
#pragma unroll
        for (int k = 0; k < BN64 / 16; ++k)
          umma_bf16_w_lead(lead, tmem + T_DXI, g_k + k * 2, HI_1024, xsj + k * 128, HI_1024, IDESC_GX,
                      (!first || k > 0) ? 1u : 0u);
        // P^T = X_s[I]^T G: M = c, N = j, K = i (128); K steps of 2 KB in both
#pragma unroll
        for (int k = 0; k < BM / 16; ++k)
          umma_bf16_w_lead(lead, tmem + T_P + b * 64, dXsI_mn + k * 128, HI_1024, g_mn + k * 128, HI_1024,
                      IDESC_PT, k > 0 ? 1u : 0u);
        umma_commit_lead(lead, P_FULL(b));
        umma_commit_lead(lead, EMPTY_S(ts));
        ++ng;
        return true;
      };
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        int u, pp;
        decode_item(p, item, u, pp);
        const Unit U = decode_unit(p, u);
        for (int pass = 0; ok && pass < item_passes(U, pp); ++pass) {
          const int I = pass_block(U, pp, pass);
          if (!(ok = mbar_wait_warp(FULL_I, nI & 1, wc, W_MMA_FULL_I))) break;
          const int nT = n_col_tiles64(p, U, I);
          int prev_ts = -1;
          for (int J = 0; J < nT; ++J) {
            const int tt = nJ & 1, ts = nJ & 3, b = ns & 1;
            if (!(ok = mbar_wait_warp(FULL_T(tt), (nJ >> 1) & 1, wc, W_MMA_FULL_J))) break;
            if (!(ok = mbar_wait_warp(S_EMPTY(b), ((ns >> 1) & 1) ^ 1, wc, W_MMA_S_EMPTY))) break;
            tc_fence_after();
            const uint32_t acc = tmem + T_S + b * 128;
            const uint32_t xtj = dXtJ_k0 + tt * J_STEP, xsj = dXsJ_k0 + ts * J_STEP;
            // K steps: 32 B within a 128 B row, then the next 64-column box
            // (16 KB apart for 128-row tiles, 8 KB for 64-row tiles)
#pragma unroll
            for (int k = 0; k < D / 16; ++k)
              umma_bf16_w_lead(lead, acc, dXtI_k + (k >> 2) * (BOX >> 4) + (k & 3) * 2, HI_1024,
                          xtj + (k >> 2) * (L::BOX_J >> 4) + (k & 3) * 2, HI_1024, IDESC_S,
                          k > 0 ? 1u : 0u);
            issued = true;
            umma_commit_lead(lead, EMPTY_T(tt));
            if (!(ok = mbar_wait_warp(FULL_S(ts), (nJ >> 2) & 1, wc, W_MMA_FULL_J))) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < D / 16; ++k)
              umma_bf16_w_lead(lead, acc + 64, dXsI_k + (k >> 2) * (BOX >> 4) + (k & 3) * 2, HI_1024,
                          xsj + (k >> 2) * (L::BOX_J >> 4) + (k & 3) * 2, HI_1024, IDESC_S,
                          k > 0 ? 1u : 0u);
            umma_commit_lead(lead, S_FULL(b));
            ++ns;
            ++nJ;
            if (prev_ts >= 0 && !(ok = grad(prev_ts, J == 1))) break;
            prev_ts = ts;
          }
          if (!ok) break;
          if (!(ok = grad(prev_ts, nT == 1))) break;
          umma_commit_lead(lead, EMPTY_I);
          umma_commit_lead(lead, DXI_FULL);
          ++nI;
          ++nrb;
        }
      }
      if (issued) {
        umma_commit_lead(lead, DRAIN);
        mbar_wait_drain(DRAIN, 0, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp >= BWD_EPI_WARP) {
    // ------------------------------------------------------- epilogue
    const int q = warp - BWD_EPI_WARP;
    const uint32_t stg = base + L::STG + q * 2 * L::STG_BYTES;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    uint32_t np = 0, nrb = 0, nstg = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      int u, pp;
        decode_item(p, item, u, pp);
      const Unit U = decode_unit(p, u);
      for (int pass = 0; ok && pass < item_passes(U, pp); ++pass) {
        const int I = pass_block(U, pp, pass);
        const int nT = n_col_tiles64(p, U, I);
        for (int J = 0; J < nT; ++J) {
          const int b = np & 1;
          ok = mbar_wait(P_FULL(b), (np >> 1) & 1, wc, W_EPI_P_FULL);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          // P^T rows are the d columns c = 32q + lane; its columns are the 64
          // rows j of column tile J.  Each 32-row half becomes one 32 x 32 box
          // of dX[J] (row j, column c), written one 128-byte row per store.
#pragma unroll 1
          for (int jb = 0; jb < 2; ++jb) {
            float v[32];
            tmem_ld32(tmem + lane_addr + T_P + b * 64 + jb * 32, v);
            tmem_wait_ld();
            if (jb == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(P_EMPTY(b));
            }
            const uint32_t buf = stg + (nstg & 1) * L::STG_BYTES;
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              st_shared_b32(buf + jj * 128 + (((lane >> 2) ^ (jj & 7)) << 4) + (lane & 3) * 4,
                            v[jj]);
            fence_proxy_async_smem();
            __syncwarp();
            const int row0 = U.tok0 + J * BN64 + jb * 32;
            if (lane == 0) {
              if (row0 < p.N) tma_reduce_add_4d(&U.seg->tm_dx, buf, q * 32, row0, U.h, U.b);
              bulk_commit();
            }
            ++nstg;
          }
          ++np;
        }
        if (!ok) break;
        ok = mbar_wait(DXI_FULL, nrb & 1, wc, W_EPI_DXI_FULL);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        epilogue_reduce<D>(tmem + lane_addr + T_DXI, stg, nstg, &U.seg->tm_dx, U.tok0 + I * BM + q * 32,
                           U.h, U.b, p.N, lane, DXI_EMPTY);
        ++nrb;
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    // --------------------------------------------------- row warpgroups
    const int q = warp & 3;
    const int wg = warp >> 2;      // 16-column slice of each 64-column tile
    const int r = q * 32 + lane;
    const float sl2 = p.sl2;
    const uint32_t row_g = r * 128;  // row r of a G buffer: 128 bytes, chunks 2wg, 2wg+1
    uint32_t ns = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      int u, pp;
        decode_item(p, item, u, pp);
      const Unit U = decode_unit(p, u);
      for (int pass = 0; ok && pass < item_passes(U, pp); ++pass) {
        const int I = pass_block(U, pp, pass);
        const int row = I * BM + r;
        const int L = U.len;
        const bool rvalid = row < L;
        float bt = 0.f, bs = 0.f, mul = 0.f;
        if (rvalid) {
          const float4 st4 = reinterpret_cast<const float4*>(U.seg->stats)[U.row0 + row];
          bt = -st4.y * kLog2e;
          bs = -st4.z * kLog2e;
          const float up = U.seg->dkl ? U.seg->dkl[U.row0 + row] : 1.0f / static_cast<float>(L);
          mul = up * p.scale;   // the logit scale of dX_s is folded into G
        }
        const int lim = !rvalid ? -1 : (p.causal ? min(row, L - 1) : L - 1);
        if (lim == 0) mul = 0.f;   // one allowed entry: R_t = R_s = 1, the gradient is 0
        const int nT = n_col_tiles64(p, U, I);
        const float2 sl2v = make_float2(sl2, sl2), btv = make_float2(bt, bt),
                     bsv = make_float2(bs, bs), mulv = make_float2(mul, mul),
                     m1 = make_float2(-1.f, -1.f);
        for (int J = 0; J < nT; ++J) {
          const int b = ns & 1;
          const uint32_t par = (ns >> 1) & 1;
          ok = mbar_wait(S_FULL(b), par, wc, W_SM_S_FULL);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + T_S + b * 128 + wg * 16;
          float t[16], s[16];
          tmem_ld16(ta, t);
          tmem_ld16(ta + 64, s);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(S_EMPTY(b));
          const int col0 = J * BN64 + wg * 16;
          const bool need_mask = !rvalid || (col0 + 15 > lim);
          uint32_t pk[8];
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            const float2 at = __ffma2_rn(make_float2(t[k], t[k + 1]), sl2v, btv);
            const float2 as = __ffma2_rn(make_float2(s[k], s[k + 1]), sl2v, bsv);
            const float2 et = ex2_approx2(at), es = ex2_approx2(as);
            float2 g = __fmul2_rn(__ffma2_rn(et, m1, es), mulv);
            if (need_mask) {
              g.x = (col0 + k <= lim) ? g.x : 0.f;
              g.y = (col0 + k + 1 <= lim) ? g.y : 0.f;
            }
            pk[k >> 1] = pack_bf16x2(g.x, g.y);
          }
          // No wait for G buffer b: the MMA warp issues the gradient MMAs of tile
          // t-2 (the last reader of this buffer) before the logit MMAs of tile t,
          // and the commit behind S_FULL covers every MMA it issued before, so
          // having seen S_FULL(t) the buffer is free.
          const uint32_t gsm = base + L::G + b * L::G_BYTES + row_g;
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int cc = 2 * wg + h2;
            st_shared_v4(gsm + ((cc ^ (r & 7)) << 4), pk[4 * h2], pk[4 * h2 + 1], pk[4 * h2 + 2],
                         pk[4 * h2 + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(G_FULL(b));
          ++ns;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == BWD_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =========================================================================
//        BACKWARD, d = 128: adjacent row-block pairs, column-tile outer
// =========================================================================
// The same mathematics again, scheduled so that the column-side product
// P^T = sum_i X_s[i]^T G[i, J] of a 64-column tile J is summed over 256 rows
// (two adjacent 128-row blocks R0 = 2k, R1 = 2k+1) in TMEM before it is added
// into dX once.  Against one 128-row block per pass this halves the f32
// reduce-adds into dX (an L2-throughput cost) and the column-tile loads per
// logit.  Tiles run in the order (R0, J), (R1, J), (R0, J+1), ...; column
// tiles that only R1 reaches under the causal mask run alone.  Two warps
// issue MMAs: one the logits of the next tile, one the gradient products of
// the tile whose G was just stored.
//   TMEM: Z_t 0..63, Z_s 64..127 (one buffer; under the causal mask the row
//         warps read Z_t, release it and form the teacher's exps while Z_s is
//         computed, and the next tile's Z_t is computed while they read Z_s;
//         the full mask reads and releases both at once), dX_R0 128..255,
//         dX_R1 256..383, P^T 2 x 64 at 384.
//   smem: X_t, X_s of R0 and R1 (4 x 32 KB); one ring of 16 KB slots for the
//         teacher and student column tiles; G; epilogue staging 4 x 4 KB.
//         Causal mask: 3 slots and G 2 x 16 KB (the row warps store tile t's
//         G while the gradient MMAs of tile t-1 read the other buffer); full
//         mask: 4 slots and G 16 KB.
// A work item is the pair sequence k = npb-1-m followed by k = m (npb row-block
// pairs per unit), which evens out the causal triangle across items.  With
// few row blocks the items are too coarse to balance 148 SMs, so sequences of
// at most 32 row blocks may use relkl_bwd_tc64_kernel instead (tc_bwd_kind).
template <bool SYM>
struct BwdPairSmem {
  static constexpr int TILE_I = BM * 128 * 2;        // 128 rows: boxes of 128 x 64 (16 KB)
  static constexpr int BOX_I = BM * 128;
  static constexpr int TILE_J = 64 * 128 * 2;        // 64 rows: boxes of 64 x 64 (8 KB)
  static constexpr int BOX_J = 64 * 128;
  static constexpr int XT_R0 = 0;
  static constexpr int XS_R0 = TILE_I;
  static constexpr int XT_R1 = 2 * TILE_I;
  static constexpr int XS_R1 = 3 * TILE_I;
  // column tiles: one ring of 16 KB slots shared by the teacher and student
  // tiles, taken in the order X_t[J], X_s[J], X_t[J+1], ... (the teacher tile
  // leaves after its logit MMAs, the student tile only after the gradient MMAs
  // of its last row block).  Causal mask: three slots and two G buffers; full
  // mask (more row-warp work per tile, where the second G buffer measured
  // slower than a fourth slot): four slots and one G buffer.
  static constexpr int NSLOT = SYM ? 4 : 3;
  static constexpr int NG = SYM ? 1 : 2;
  static constexpr int RING = 4 * TILE_I;
  static constexpr int G = RING + NSLOT * TILE_J;    // NG x (128 x 64 bf16)
  static constexpr int G_BYTES = BM * 64 * 2;
  static constexpr int STG = G + NG * G_BYTES;       // 4 warps x one 32 x 32 f32 box
  static constexpr int STG_BYTES = 32 * 32 * 4;
  static constexpr int BARS = STG + 4 * STG_BYTES;
  // full_I, empty_I, slot_full[NSLOT], slot_empty[NSLOT], s_full, s_empty,
  // g_full[NG], g_empty[NG], p_full[2], p_empty[2], dxi_full, dxi_empty,
  // drain x 2, t_full, t_empty
  static constexpr int B_SLOT_FULL = 2, B_SLOT_EMPTY = 2 + NSLOT, B_S = 2 + 2 * NSLOT;
  static constexpr int B_G_FULL = B_S + 2, B_G_EMPTY = B_G_FULL + NG, B_P = B_G_EMPTY + NG;
  static constexpr int B_REST = B_P + 4;
  static constexpr int NBAR = B_REST + 6;
  static constexpr int MISC = BARS + NBAR * 8;
  static constexpr int BYTES = MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
};
static_assert(BwdPairSmem<false>::ALLOC <= 232448 && BwdPairSmem<true>::ALLOC <= 232448,
              "backward shared memory exceeds 227 KB");
// warps 0-15 row, 16-19 epilogue, 20 TMA, 21 logit MMAs, 22 gradient MMAs
constexpr int BWDP_THREADS = 736;
// Causal masks at d = 128: sequences of more than 32 row blocks always take the
// paired-block kernel, sequences of fewer than 16 the one-block kernel, and in
// between the launch estimates both (tc_bwd_kind).
constexpr int kPairAlwaysBlocks = 33, kPairMinBlocks = 16;
constexpr int BWDP_LOGIT_WARP = 21, BWDP_GRAD_WARP = 22;

// Sequence `which` (0 or 1) of pair item m: its first row block, or -1.
__host__ __device__ __forceinline__ int pair_seq_block(const Unit& U, int m, int which) {
  const int npb = (U.nblk + 1) / 2;
  if (m >= (npb + 1) / 2) return -1;   // past a short packed sequence's items
  const int k = which == 0 ? npb - 1 - m : m;
  if (which == 1 && k == npb - 1 - m) return -1;
  return 2 * k;
}

template <bool SYM>
__global__ void __launch_bounds__(BWDP_THREADS, 1)
relkl_bwd_pair_kernel(const __grid_constant__ TcParams p) {
  using L = BwdPairSmem<SYM>;
  constexpr int D = 128;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t bar0 = base + L::BARS;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * i; };
  const uint32_t FULL_I = BAR(0), EMPTY_I = BAR(1);
  // ring use u (X_t[J] of the n-th column tile: u = 2n, X_s[J]: u = 2n + 1) sits
  // in slot u % NSLOT and is that slot's (u / NSLOT)-th fill
  auto SLOT_FULL = [&](uint32_t u) { return BAR(L::B_SLOT_FULL + static_cast<int>(u % L::NSLOT)); };
  auto SLOT_EMPTY = [&](uint32_t u) { return BAR(L::B_SLOT_EMPTY + static_cast<int>(u % L::NSLOT)); };
  auto SLOT_PAR = [&](uint32_t u) { return (u / L::NSLOT) & 1u; };
  const uint32_t S_FULL = BAR(L::B_S), S_EMPTY = BAR(L::B_S + 1);
  // tile t's G goes to buffer t % NG, that buffer's (t / NG)-th fill
  auto G_FULL = [&](uint32_t t) { return BAR(L::B_G_FULL + static_cast<int>(t % L::NG)); };
  auto G_EMPTY = [&](uint32_t t) { return BAR(L::B_G_EMPTY + static_cast<int>(t % L::NG)); };
  auto G_PAR = [&](uint32_t t) { return (t / L::NG) & 1u; };
  auto P_FULL = [&](int b) { return BAR(L::B_P + b); };
  auto P_EMPTY = [&](int b) { return BAR(L::B_P + 2 + b); };
  const uint32_t DXI_FULL = BAR(L::B_REST), DXI_EMPTY = BAR(L::B_REST + 1);
  const uint32_t DRAIN_L = BAR(L::B_REST + 2), DRAIN_G = BAR(L::B_REST + 3);
  // causal mask: T_FULL / T_EMPTY guard Z_t, S_FULL / S_EMPTY Z_s; full mask:
  // S_FULL / S_EMPTY guard both
  const uint32_t T_FULL = BAR(L::B_REST + 4), T_EMPTY = BAR(L::B_REST + 5);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::MISC + 4);

  WaitCtl wc{p.status, abort_flag, p.timeout_ns};
  constexpr uint32_t T_S = 0, T_DX0 = 128, T_P = 384;
  static_assert(T_S + 2 * BN64 <= T_DX0 && T_DX0 + 2 * D <= T_P && T_P + 2 * BN64 <= 512,
                "TMEM columns: Z_t, Z_s | dX_R0, dX_R1 | 2 x P^T");

  if (threadIdx.x == 0) {
    mbar_init(FULL_I, 1);
    mbar_init(EMPTY_I, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(P_FULL(s), 1);
      mbar_init(P_EMPTY(s), 4);
    }
    for (uint32_t b = 0; b < L::NG; ++b) {
      mbar_init(G_FULL(b), 16);
      mbar_init(G_EMPTY(b), 1);
    }
    for (uint32_t u = 0; u < L::NSLOT; ++u) {
      mbar_init(SLOT_FULL(u), 1);
      mbar_init(SLOT_EMPTY(u), 1);
    }
    mbar_init(S_FULL, 1);
    mbar_init(S_EMPTY, 16);
    mbar_init(T_FULL, 1);
    mbar_init(T_EMPTY, 16);
    mbar_init(DXI_FULL, 1);
    mbar_init(DXI_EMPTY, 4);
    mbar_init(DRAIN_L, 1);
    mbar_init(DRAIN_G, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == BWDP_LOGIT_WARP) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == BWD_TMA_WARP) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      for (int s = 0; s < p.n_seg; ++s) {
        tma_prefetch_desc(&p.seg[s].tm_t);
        tma_prefetch_desc(&p.seg[s].tm_s);
        tma_prefetch_desc(&p.seg[s].tm_t64);
        tma_prefetch_desc(&p.seg[s].tm_s64);
        tma_prefetch_desc(&p.seg[s].tm_dx);
      }
      uint32_t nseq = 0, nJ = 0;
      uint32_t arms[L::NSLOT] = {};
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        int u, m;
        decode_item(p, item, u, m);
        const Unit U = decode_unit(p, u);
        for (int w = 0; ok && w < 2; ++w) {
          const int R0 = pair_seq_block(U, m, w);
          if (R0 < 0) break;
          const bool has1 = R0 + 1 < U.nblk;
          if (!(ok = mbar_wait(EMPTY_I, (nseq & 1) ^ 1, wc, W_TMA_EMPTY_I))) break;
          mbar_arrive_expect_tx(FULL_I, (has1 ? 4 : 2) * L::TILE_I);
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            tma_load_4d(base + L::XT_R0 + b * L::BOX_I, &U.seg->tm_t, FULL_I, b * 64, U.tok0 + R0 * BM, U.h, U.b);
            tma_load_4d(base + L::XS_R0 + b * L::BOX_I, &U.seg->tm_s, FULL_I, b * 64, U.tok0 + R0 * BM, U.h, U.b);
            if (has1) {
              tma_load_4d(base + L::XT_R1 + b * L::BOX_I, &U.seg->tm_t, FULL_I, b * 64, U.tok0 + (R0 + 1) * BM,
                          U.h, U.b);
              tma_load_4d(base + L::XS_R1 + b * L::BOX_I, &U.seg->tm_s, FULL_I, b * 64, U.tok0 + (R0 + 1) * BM,
                          U.h, U.b);
            }
          }
          ++nseq;
          const int nT = n_col_tiles64_s<SYM>(p, U, has1 ? R0 + 1 : R0);
          for (int J = 0; J < nT; ++J) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {   // X_t[J], then X_s[J]
              const uint32_t use = 2 * nJ + which;
              const uint32_t slot = use % L::NSLOT;
              if (!(ok = mbar_wait(SLOT_EMPTY(use), SLOT_PAR(use) ^ 1, wc, W_TMA_EMPTY_J))) break;
              mbar_arrive_expect_tx(SLOT_FULL(use), L::TILE_J);
#pragma unroll
              for (int b = 0; b < 2; ++b)
                tma_load_4d(base + L::RING + slot * L::TILE_J + b * L::BOX_J,
                            which ? &U.seg->tm_s64 : &U.seg->tm_t64, SLOT_FULL(use), b * 64,
                            U.tok0 + J * BN64, U.h, U.b);
              ++arms[slot];
            }
            if (!ok) break;
            ++nJ;
          }
        }
      }
      if (nseq) mbar_wait_drain(FULL_I, (nseq - 1) & 1, kDrainNs);
      for (uint32_t k = 0; k < L::NSLOT; ++k)
        if (arms[k]) mbar_wait_drain(SLOT_FULL(k), (arms[k] - 1) & 1, kDrainNs);
    }
    __syncwarp();
  } else if (warp == BWDP_LOGIT_WARP || warp == BWDP_GRAD_WARP) {
    // ------------------------------------------------------------ MMA
    // Two issuing warps share the tensor pipe: one issues the logit MMAs of
    // tile t+1 as soon as the row warps have read tile t's logits, the other
    // the gradient MMAs of tile t once its G is stored, so that neither
    // waits behind the other's barriers.  Each warp runs its loop converged
    // (descriptor words stay warp-uniform); one elected lane issues.
    const bool is_logit = warp == BWDP_LOGIT_WARP;
    const uint32_t lead = elect_leader();
    constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN64, 0, 0);
    constexpr uint32_t IDESC_GX = idesc_bf16_f32(BM, D, 0, 1);    // A = G (K-major), B = X_s[J] (MN)
    constexpr uint32_t IDESC_PT = idesc_bf16_f32(D, BN64, 1, 1);  // A = X_s[R]^T (MN), B = G (MN)
    const uint32_t HI_1024 = sw128_desc_hi(1024);
    const uint32_t dXtR_k[2] = {sw128_desc_lo(base + L::XT_R0, 16), sw128_desc_lo(base + L::XT_R1, 16)};
    const uint32_t dXsR_k[2] = {sw128_desc_lo(base + L::XS_R0, 16), sw128_desc_lo(base + L::XS_R1, 16)};
    const uint32_t dXsR_mn[2] = {sw128_desc_lo(base + L::XS_R0, L::BOX_I),
                                 sw128_desc_lo(base + L::XS_R1, L::BOX_I)};
    const uint32_t dRing_k0 = sw128_desc_lo(base + L::RING, 16);
    const uint32_t dRing_mn0 = sw128_desc_lo(base + L::RING, L::BOX_J);
    const uint32_t dG_k = sw128_desc_lo(base + L::G, 16);
    const uint32_t dG_mn = sw128_desc_lo(base + L::G, L::G_BYTES);
    constexpr uint32_t J_STEP = L::TILE_J >> 4, G_STEP = L::G_BYTES >> 4;
    uint32_t nseq = 0, nJ = 0, nt = 0, np = 0;
    bool ok = true, issued = false;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      int u, m;
      decode_item(p, item, u, m);
      const Unit U = decode_unit(p, u);
      for (int w = 0; ok && w < 2; ++w) {
        const int R0 = pair_seq_block(U, m, w);
        if (R0 < 0) break;
        const bool has1 = R0 + 1 < U.nblk;
        const int nT0 = n_col_tiles64_s<SYM>(p, U, R0);
        const int nT = has1 ? n_col_tiles64_s<SYM>(p, U, R0 + 1) : nT0;
        if (!(ok = mbar_wait_warp(FULL_I, nseq & 1, wc, W_MMA_FULL_I))) break;
        bool first_seq = true;
        for (int J = 0; ok && J < nT; ++J) {
          const uint32_t ut = 2 * nJ, us = 2 * nJ + 1;   // ring uses of X_t[J], X_s[J]
          for (int rs = 0; rs < 2; ++rs) {
            if (rs == 0 && J >= nT0) continue;
            if (rs == 1 && !has1) continue;
            const bool first_p = rs == 0 || J >= nT0;
            const bool last_p = rs == 1 || !has1;
            if (is_logit) {
              // Z_t, Z_s of tile (R, J) into the logit buffer; under the causal mask
              // Z_t as soon as the row warps have read the previous Z_t, Z_s once
              // they have read the previous Z_s
              if (!(ok = mbar_wait_warp(SLOT_FULL(ut), SLOT_PAR(ut), wc, W_MMA_FULL_J))) break;
              if (!(ok = mbar_wait_warp(SYM ? S_EMPTY : T_EMPTY, (nt & 1) ^ 1, wc, W_MMA_S_EMPTY)))
                break;
              tc_fence_after();
              const uint32_t xtj = dRing_k0 + (ut % L::NSLOT) * J_STEP;
              const uint32_t xsj = dRing_k0 + (us % L::NSLOT) * J_STEP;
              // K steps: 32 B within a 128 B row, then the next 64-column box
#pragma unroll
              for (int k = 0; k < D / 16; ++k)
                umma_bf16_w_lead(lead, tmem + T_S, dXtR_k[rs] + (k >> 2) * (L::BOX_I >> 4) + (k & 3) * 2,
                                 HI_1024, xtj + (k >> 2) * (L::BOX_J >> 4) + (k & 3) * 2, HI_1024,
                                 IDESC_S, k > 0 ? 1u : 0u);
              issued = true;
              if (last_p) umma_commit_lead(lead, SLOT_EMPTY(ut));
              if (!SYM) umma_commit_lead(lead, T_FULL);
              if (!(ok = mbar_wait_warp(SLOT_FULL(us), SLOT_PAR(us), wc, W_MMA_FULL_J))) break;
              if (!SYM && !(ok = mbar_wait_warp(S_EMPTY, (nt & 1) ^ 1, wc, W_MMA_S_EMPTY))) break;
              tc_fence_after();
#pragma unroll
              for (int k = 0; k < D / 16; ++k)
                umma_bf16_w_lead(lead, tmem + T_S + 64, dXsR_k[rs] + (k >> 2) * (L::BOX_I >> 4) + (k & 3) * 2,
                                 HI_1024, xsj + (k >> 2) * (L::BOX_J >> 4) + (k & 3) * 2, HI_1024,
                                 IDESC_S, k > 0 ? 1u : 0u);
              umma_commit_lead(lead, S_FULL);
            } else {
              // dX_R += G X_s[J] and P^T (+)= X_s[R]^T G for tile (R, J).  G_FULL
              // implies the tile's logits (hence its column tiles) are complete.
              const int pb = np & 1;
              const uint32_t gb = nt % L::NG;
              if (!(ok = mbar_wait_warp(G_FULL(nt), G_PAR(nt), wc, W_MMA_G_FULL))) break;
              if (first_p && !(ok = mbar_wait_warp(P_EMPTY(pb), ((np >> 1) & 1) ^ 1, wc, W_MMA_P_EMPTY)))
                break;
              if (first_seq && !(ok = mbar_wait_warp(DXI_EMPTY, (nseq & 1) ^ 1, wc, W_MMA_DXI_EMPTY)))
                break;
              first_seq = false;
              tc_fence_after();
              const uint32_t xsj = dRing_mn0 + (us % L::NSLOT) * J_STEP;
              const uint32_t gk = dG_k + gb * G_STEP, gmn = dG_mn + gb * G_STEP;
              // M = i, N = c, K = j (64); K steps of 32 B (G) and 2 KB (X_s[J])
#pragma unroll
              for (int k = 0; k < BN64 / 16; ++k)
                umma_bf16_w_lead(lead, tmem + T_DX0 + rs * 128, gk + k * 2, HI_1024, xsj + k * 128,
                                 HI_1024, IDESC_GX, (J > 0 || k > 0) ? 1u : 0u);
              // M = c, N = j, K = i (128); K steps of 2 KB in both
#pragma unroll
              for (int k = 0; k < BM / 16; ++k)
                umma_bf16_w_lead(lead, tmem + T_P + pb * 64, dXsR_mn[rs] + k * 128, HI_1024,
                                 gmn + k * 128, HI_1024, IDESC_PT, (!first_p || k > 0) ? 1u : 0u);
              issued = true;
              umma_commit_lead(lead, G_EMPTY(nt));
              if (last_p) {
                umma_commit_lead(lead, P_FULL(pb));
                umma_commit_lead(lead, SLOT_EMPTY(us));
                ++np;
              }
            }
            ++nt;
          }
          ++nJ;
        }
        if (!ok) break;
        if (!is_logit) {
          umma_commit_lead(lead, EMPTY_I);
          umma_commit_lead(lead, DXI_FULL);
        }
        ++nseq;
      }
    }
    if (issued) {
      const uint32_t drain = is_logit ? DRAIN_L : DRAIN_G;
      umma_commit_lead(lead, drain);
      mbar_wait_drain(drain, 0, kDrainNs);
    }
    __syncwarp();
  } else if (warp >= BWD_EPI_WARP) {
    // ------------------------------------------------------- epilogue
    // Every f32 addition into dX goes out as a TMA reduce-add of a 32 x 32
    // box staged in this warp's 4 KB of shared memory (128-byte swizzle).
    // P^T lane c = 32q + lane holds dX[J*64 + j][c] for the tile's 64 columns
    // j, so it is staged transposed: one 128-byte row of the box per j.
    const int q = warp - BWD_EPI_WARP;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t stg = base + L::STG + q * L::STG_BYTES;
    uint32_t np = 0, nseq = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      int u, m;
        decode_item(p, item, u, m);
      const Unit U = decode_unit(p, u);
      for (int w = 0; ok && w < 2; ++w) {
        const int R0 = pair_seq_block(U, m, w);
        if (R0 < 0) break;
        const bool has1 = R0 + 1 < U.nblk;
        const int nT = n_col_tiles64_s<SYM>(p, U, has1 ? R0 + 1 : R0);
        for (int J = 0; J < nT; ++J) {
          const int b = np & 1;
          ok = mbar_wait(P_FULL(b), (np >> 1) & 1, wc, W_EPI_P_FULL);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int jb = 0; jb < 2; ++jb) {
            float v[32];
            tmem_ld32(tmem + lane_addr + T_P + b * 64 + jb * 32, v);
            tmem_wait_ld();
            if (jb == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(P_EMPTY(b));
            }
            if (lane == 0) bulk_wait_read<0>();   // the previous box has left the buffer
            __syncwarp();
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              st_shared_b32(stg + jj * 128 + (((lane >> 2) ^ (jj & 7)) << 4) + (lane & 3) * 4, v[jj]);
            fence_proxy_async_smem();
            __syncwarp();
            const int row0 = U.tok0 + J * BN64 + jb * 32;
            if (lane == 0) {
              if (row0 < p.N) tma_reduce_add_4d(&U.seg->tm_dx, stg, q * 32, row0, U.h, U.b);
              bulk_commit();
            }
          }
          ++np;
        }
        if (!ok) break;
        // dX rows of the pair: lane = row, 32-column boxes
        ok = mbar_wait(DXI_FULL, nseq & 1, wc, W_EPI_DXI_FULL);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        for (int rs = 0; rs < 2; ++rs) {
          const int row0 = U.tok0 + (R0 + rs) * BM + q * 32;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float v[32];
            tmem_ld32(tmem + lane_addr + T_DX0 + rs * 128 + c * 32, v);
            tmem_wait_ld();
            if (rs == 1 && c == D / 32 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(DXI_EMPTY);
            }
            if (rs == 1 && !has1) continue;
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
            const uint32_t rowp = stg + lane * 128;
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4)
              st_shared_v4(rowp + ((k4 ^ (lane & 7)) << 4), __float_as_uint(v[4 * k4]),
                           __float_as_uint(v[4 * k4 + 1]), __float_as_uint(v[4 * k4 + 2]),
                           __float_as_uint(v[4 * k4 + 3]));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (row0 < p.N) tma_reduce_add_4d(&U.seg->tm_dx, stg, c * 32, row0, U.h, U.b);
              bulk_commit();
            }
          }
        }
        ++nseq;
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    // --------------------------------------------------- row warpgroups
    const int q = warp & 3;
    const int wg = warp >> 2;      // 16-column slice of each 64-column tile
    const int r = q * 32 + lane;
    const float sl2 = p.sl2;
    const uint32_t gsm0 = base + L::G + r * 128;  // row r of G: 128 bytes, chunks 2wg, 2wg+1
    uint32_t nt = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      int u, m;
        decode_item(p, item, u, m);
      const Unit U = decode_unit(p, u);
      for (int w = 0; ok && w < 2; ++w) {
        const int R0 = pair_seq_block(U, m, w);
        if (R0 < 0) break;
        const bool has1 = R0 + 1 < U.nblk;
        const int nT0 = n_col_tiles64_s<SYM>(p, U, R0);
        const int nT = has1 ? n_col_tiles64_s<SYM>(p, U, R0 + 1) : nT0;
        const int L = U.len;
        // per-row constants of both row blocks
        float bt[2], bs[2], mul[2];
        int lim[2];
#pragma unroll
        for (int rs = 0; rs < 2; ++rs) {
          const int row = (R0 + rs) * BM + r;
          const bool rvalid = row < L && (rs == 0 || has1);
          bt[rs] = bs[rs] = mul[rs] = 0.f;
          if (rvalid) {
            const float4 st4 = reinterpret_cast<const float4*>(U.seg->stats)[U.row0 + row];
            bt[rs] = -st4.y * kLog2e;
            bs[rs] = -st4.z * kLog2e;
            const float up = U.seg->dkl ? U.seg->dkl[U.row0 + row] : 1.0f / static_cast<float>(L);
            mul[rs] = up * p.scale;   // the logit scale of dX_s is folded into G
          }
          lim[rs] = !rvalid ? -1 : (p.causal ? min(row, L - 1) : L - 1);
          if (lim[rs] == 0) mul[rs] = 0.f;   // one allowed entry: R_t = R_s = 1, the gradient is 0
        }
        const float2 sl2v = make_float2(sl2, sl2), m1 = make_float2(-1.f, -1.f);
        for (int J = 0; ok && J < nT; ++J) {
          for (int rs = 0; rs < 2; ++rs) {
            if (rs == 0 && J >= nT0) continue;
            if (rs == 1 && !has1) continue;
            // full mask, off the diagonal block: each lane fetches the partner
            // constants of one of this warpgroup's 16 columns while the logits
            // are still being computed
            const bool off = SYM && J < 2 * (R0 + rs);
            PartnerCol pc{0.f, 0.f, 0.f};
            if (off) pc = partner_column(U, p, J * BN64 + wg * 16 + (lane & 15));
            ok = mbar_wait(SYM ? S_FULL : T_FULL, nt & 1, wc, W_SM_S_FULL);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + T_S + wg * 16;
            float t[16], s[16];
            tmem_ld16(ta, t);
            if constexpr (SYM) tmem_ld16(ta + 64, s);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(SYM ? S_EMPTY : T_EMPTY);
            const float btr = rs ? bt[1] : bt[0], bsr = rs ? bs[1] : bs[0];
            const float mr = rs ? mul[1] : mul[0];
            const int limr = rs ? lim[1] : lim[0];
            const float2 btv = make_float2(btr, btr), bsv = make_float2(bsr, bsr),
                         mulv = make_float2(mr, mr);
            const int col0 = J * BN64 + wg * 16;
            if constexpr (!SYM) {
              // the teacher's exps while Z_s is still being computed (t then holds
              // e_t), then Z_s
#pragma unroll
              for (int k = 0; k < 16; k += 2) {
                const float2 et = ex2_approx2(__ffma2_rn(make_float2(t[k], t[k + 1]), sl2v, btv));
                t[k] = et.x;
                t[k + 1] = et.y;
              }
              ok = mbar_wait(S_FULL, nt & 1, wc, W_SM_S_FULL);
              ok = __all_sync(0xffffffffu, ok);
              if (!ok) break;
              tc_fence_after();
              tmem_ld16(ta + 64, s);
              tmem_wait_ld();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(S_EMPTY);
            }
            if constexpr (SYM) {
              // full mask: tiles of the diagonal block carry G itself, the others
              // G plus its transposed partner (4 exps per entry); as in the causal
              // path the G buffer is awaited only once the entries are formed
              uint32_t pk[8];
              PartnerTile pt{1.f, 1.f, false};
              if (off) pt = partner_tile(pc, btr, bsr);
              form_g_pack<16>(t, s, btr, bsr, mr, col0, limr, off, pc, pt, 0, p, pk);
              // the gradient MMAs of NG tiles back have read this G buffer
              ok = mbar_wait(G_EMPTY(nt), G_PAR(nt) ^ 1, wc, W_SM_G_EMPTY);
              ok = __all_sync(0xffffffffu, ok);
              if (!ok) break;
              const uint32_t gsm = gsm0 + (nt % L::NG) * L::G_BYTES;
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                const int cc = 2 * wg + h2;  // 16-byte chunk within the 128-byte row
                st_shared_v4(gsm + ((cc ^ (r & 7)) << 4), pk[4 * h2], pk[4 * h2 + 1],
                             pk[4 * h2 + 2], pk[4 * h2 + 3]);
              }
            } else {
            const bool need_mask = col0 + 15 > limr;
            uint32_t pk[8];
#pragma unroll
            for (int k = 0; k < 16; k += 2) {
              const float2 es = ex2_approx2(__ffma2_rn(make_float2(s[k], s[k + 1]), sl2v, bsv));
              float2 g = __fmul2_rn(__ffma2_rn(make_float2(t[k], t[k + 1]), m1, es), mulv);
              if (need_mask) {
                g.x = (col0 + k <= limr) ? g.x : 0.f;
                g.y = (col0 + k + 1 <= limr) ? g.y : 0.f;
              }
              pk[k >> 1] = pack_bf16x2(g.x, g.y);
            }
            // the gradient MMAs of NG tiles back have read this G buffer
            ok = mbar_wait(G_EMPTY(nt), G_PAR(nt) ^ 1, wc, W_SM_G_EMPTY);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const uint32_t gsm = gsm0 + (nt % L::NG) * L::G_BYTES;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int cc = 2 * wg + h2;  // 16-byte chunk within the 128-byte row
              st_shared_v4(gsm + ((cc ^ (r & 7)) << 4), pk[4 * h2], pk[4 * h2 + 1], pk[4 * h2 + 2],
                           pk[4 * h2 + 3]);
            }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(G_FULL(nt));
            ++nt;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == BWDP_LOGIT_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =========================================================================
//        BACKWARD, d = 64: adjacent row-block pairs, 128-column tiles
// =========================================================================
// The paired-block schedule of relkl_bwd_pair_kernel at head dimension 64.
// The accumulators are half as wide as at d = 128, which leaves TMEM room for
// 128-column logit tiles (full-rate N = 128 logit MMAs).  The column-side
// product is formed as P = G^T X_s[R] (M = 128 columns j, N = d = 64,
// K = the rows of R0 then R1), so it is summed over both row blocks in TMEM
// and its TMEM lanes are the rows j of dX[J]: the epilogue stages them row by
// row, without a transpose.  With 64-dimensional rows the exp work per entry
// is what bounds this kernel (2 ex2 per entry against 0.08 clk of MMA work),
// so one logit buffer suffices: the next tile's logit MMAs finish while the
// row warps run the current tile's exps.  G is double-buffered, so the row
// warps never wait for the previous tile's gradient MMAs before storing.
//   TMEM: Z_t 0..127, Z_s 128..255, dX_R0 256..319, dX_R1 320..383,
//         P 2 x 64 at 384.
//   smem: X_t, X_s of R0 and R1 (4 x 16 KB); teacher and student column
//         rings 2 x 16 KB each; G 2 x 32 KB (two 64-column boxes each);
//         epilogue staging 4 x 4 KB.
struct BwdPair64Smem {
  static constexpr int TILE = BM * 64 * 2;           // 128 rows x 64 bf16: one box (16 KB)
  static constexpr int XT_R0 = 0;
  static constexpr int XS_R0 = TILE;
  static constexpr int XT_R1 = 2 * TILE;
  static constexpr int XS_R1 = 3 * TILE;
  static constexpr int XT_J = 4 * TILE;              // 2 stages
  static constexpr int XS_J = XT_J + 2 * TILE;       // 2 stages
  static constexpr int G = XS_J + 2 * TILE;          // 2 x (128 x 128 bf16, boxes of 64 columns)
  static constexpr int G_BYTES = 2 * TILE;
  static constexpr int STG = G + 2 * G_BYTES;        // 4 warps x one 32 x 32 f32 box
  static constexpr int STG_BYTES = 32 * 32 * 4;
  static constexpr int BARS = STG + 4 * STG_BYTES;
  // full_I, empty_I, fullT[2], emptyT[2], fullS[2], emptyS[2], s_full, s_empty,
  // g_full[0], g_empty[0], p_full[2], p_empty[2], dxi_full, dxi_empty, drain x 2,
  // g_full[1], g_empty[1]
  static constexpr int NBAR = 24;
  static constexpr int MISC = BARS + NBAR * 8;
  static constexpr int BYTES = MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
};
static_assert(BwdPair64Smem::ALLOC <= 232448, "backward shared memory exceeds 227 KB");

template <bool SYM>
__global__ void __launch_bounds__(BWDP_THREADS, 1)
relkl_bwd_pair64_kernel(const __grid_constant__ TcParams p) {
  using L = BwdPair64Smem;
  constexpr int D = 64;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t bar0 = base + L::BARS;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * i; };
  const uint32_t FULL_I = BAR(0), EMPTY_I = BAR(1);
  auto FULL_T = [&](int s) { return BAR(2 + s); };
  auto EMPTY_T = [&](int s) { return BAR(4 + s); };
  auto FULL_S = [&](int s) { return BAR(6 + s); };
  auto EMPTY_S = [&](int s) { return BAR(8 + s); };
  const uint32_t S_FULL = BAR(10), S_EMPTY = BAR(11);
  // G is double-buffered: the row warps store tile t's G while the gradient
  // MMAs of tile t-1 still read the other buffer
  auto G_FULL = [&](int b) { return b ? BAR(22) : BAR(12); };
  auto G_EMPTY = [&](int b) { return b ? BAR(23) : BAR(13); };
  auto P_FULL = [&](int b) { return BAR(14 + b); };
  auto P_EMPTY = [&](int b) { return BAR(16 + b); };
  const uint32_t DXI_FULL = BAR(18), DXI_EMPTY = BAR(19), DRAIN_L = BAR(20), DRAIN_G = BAR(21);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::MISC + 4);

  WaitCtl wc{p.status, abort_flag, p.timeout_ns};
  constexpr uint32_t T_S = 0, T_DX0 = 256, T_P = 384;
  static_assert(T_S + 2 * BN <= T_DX0 && T_DX0 + 2 * D <= T_P && T_P + 2 * D <= 512,
                "TMEM columns: Z_t, Z_s | dX_R0, dX_R1 | 2 x P");

  if (threadIdx.x == 0) {
    mbar_init(FULL_I, 1);
    mbar_init(EMPTY_I, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(FULL_T(s), 1);
      mbar_init(EMPTY_T(s), 1);
      mbar_init(FULL_S(s), 1);
      mbar_init(EMPTY_S(s), 1);
      mbar_init(P_FULL(s), 1);
      mbar_init(P_EMPTY(s), 4);
    }
    mbar_init(S_FULL, 1);
    mbar_init(S_EMPTY, 16);
    for (int b = 0; b < 2; ++b) {
      mbar_init(G_FULL(b), 16);
      mbar_init(G_EMPTY(b), 1);
    }
    mbar_init(DXI_FULL, 1);
    mbar_init(DXI_EMPTY, 4);
    mbar_init(DRAIN_L, 1);
    mbar_init(DRAIN_G, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == BWDP_LOGIT_WARP) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == BWD_TMA_WARP) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      for (int s = 0; s < p.n_seg; ++s) {
        tma_prefetch_desc(&p.seg[s].tm_t);
        tma_prefetch_desc(&p.seg[s].tm_s);
        tma_prefetch_desc(&p.seg[s].tm_dx);
      }
      uint32_t nseq = 0, nJ = 0;
      uint32_t armsT[2] = {0, 0}, armsS[2] = {0, 0};
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        int u, m;
        decode_item(p, item, u, m);
        const Unit U = decode_unit(p, u);
        for (int w = 0; ok && w < 2; ++w) {
          const int R0 = pair_seq_block(U, m, w);
          if (R0 < 0) break;
          const bool has1 = R0 + 1 < U.nblk;
          if (!(ok = mbar_wait(EMPTY_I, (nseq & 1) ^ 1, wc, W_TMA_EMPTY_I))) break;
          mbar_arrive_expect_tx(FULL_I, (has1 ? 4 : 2) * L::TILE);
          tma_load_4d(base + L::XT_R0, &U.seg->tm_t, FULL_I, 0, U.tok0 + R0 * BM, U.h, U.b);
          tma_load_4d(base + L::XS_R0, &U.seg->tm_s, FULL_I, 0, U.tok0 + R0 * BM, U.h, U.b);
          if (has1) {
            tma_load_4d(base + L::XT_R1, &U.seg->tm_t, FULL_I, 0, U.tok0 + (R0 + 1) * BM, U.h, U.b);
            tma_load_4d(base + L::XS_R1, &U.seg->tm_s, FULL_I, 0, U.tok0 + (R0 + 1) * BM, U.h, U.b);
          }
          ++nseq;
          const int nT = n_col_tiles_s<SYM>(p, U, has1 ? R0 + 1 : R0);
          for (int J = 0; J < nT; ++J) {
            const int st = nJ & 1;
            if (!(ok = mbar_wait(EMPTY_T(st), ((nJ >> 1) & 1) ^ 1, wc, W_TMA_EMPTY_J))) break;
            mbar_arrive_expect_tx(FULL_T(st), L::TILE);
            tma_load_4d(base + L::XT_J + st * L::TILE, &U.seg->tm_t, FULL_T(st), 0,
                        U.tok0 + J * BN, U.h, U.b);
            ++armsT[st];
            if (!(ok = mbar_wait(EMPTY_S(st), ((nJ >> 1) & 1) ^ 1, wc, W_TMA_EMPTY_J))) break;
            mbar_arrive_expect_tx(FULL_S(st), L::TILE);
            tma_load_4d(base + L::XS_J + st * L::TILE, &U.seg->tm_s, FULL_S(st), 0,
                        U.tok0 + J * BN, U.h, U.b);
            ++armsS[st];
            ++nJ;
          }
        }
      }
      if (nseq) mbar_wait_drain(FULL_I, (nseq - 1) & 1, kDrainNs);
      for (int s = 0; s < 2; ++s) {
        if (armsT[s]) mbar_wait_drain(FULL_T(s), (armsT[s] - 1) & 1, kDrainNs);
        if (armsS[s]) mbar_wait_drain(FULL_S(s), (armsS[s] - 1) & 1, kDrainNs);
      }
    }
    __syncwarp();
  } else if (warp == BWDP_LOGIT_WARP || warp == BWDP_GRAD_WARP) {
    // ------------------------------------------------------------ MMA
    // One warp issues the logit MMAs of the next tile as soon as the row
    // warps have read the current one; the other the gradient MMAs of the
    // tile whose G was just stored.  Each runs its loop converged; one
    // elected lane issues.
    const bool is_logit = warp == BWDP_LOGIT_WARP;
    const uint32_t lead = elect_leader();
    constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, 0, 0);
    constexpr uint32_t IDESC_GX = idesc_bf16_f32(BM, D, 0, 1);   // A = G (K-major), B = X_s[J] (MN)
    constexpr uint32_t IDESC_P = idesc_bf16_f32(BM, D, 1, 1);    // A = G^T (MN), B = X_s[R] (MN)
    const uint32_t HI_1024 = sw128_desc_hi(1024);
    const uint32_t dXtR_k[2] = {sw128_desc_lo(base + L::XT_R0, 16), sw128_desc_lo(base + L::XT_R1, 16)};
    const uint32_t dXsR_k[2] = {sw128_desc_lo(base + L::XS_R0, 16), sw128_desc_lo(base + L::XS_R1, 16)};
    const uint32_t dXsR_mn[2] = {sw128_desc_lo(base + L::XS_R0, L::TILE),
                                 sw128_desc_lo(base + L::XS_R1, L::TILE)};
    const uint32_t dXtJ_k0 = sw128_desc_lo(base + L::XT_J, 16);
    const uint32_t dXsJ_k0 = sw128_desc_lo(base + L::XS_J, 16);
    const uint32_t dXsJ_mn0 = sw128_desc_lo(base + L::XS_J, L::TILE);
    const uint32_t dG_k = sw128_desc_lo(base + L::G, 16);
    const uint32_t dG_mn = sw128_desc_lo(base + L::G, L::TILE);
    constexpr uint32_t J_STEP = L::TILE >> 4, BOX_STEP = L::TILE >> 4, G_STEP = L::G_BYTES >> 4;
    uint32_t nseq = 0, nJ = 0, nt = 0, np = 0;
    bool ok = true, issued = false;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      int u, m;
      decode_item(p, item, u, m);
      const Unit U = decode_unit(p, u);
      for (int w = 0; ok && w < 2; ++w) {
        const int R0 = pair_seq_block(U, m, w);
        if (R0 < 0) break;
        const bool has1 = R0 + 1 < U.nblk;
        const int nT0 = n_col_tiles_s<SYM>(p, U, R0);
        const int nT = has1 ? n_col_tiles_s<SYM>(p, U, R0 + 1) : nT0;
        if (!(ok = mbar_wait_warp(FULL_I, nseq & 1, wc, W_MMA_FULL_I))) break;
        bool first_seq = true;
        for (int J = 0; ok && J < nT; ++J) {
          const int st = nJ & 1;
          for (int rs = 0; rs < 2; ++rs) {
            if (rs == 0 && J >= nT0) continue;
            if (rs == 1 && !has1) continue;
            const bool first_p = rs == 0 || J >= nT0;
            const bool last_p = rs == 1 || !has1;
            if (is_logit) {
              // Z_t, Z_s of tile (R, J): M = 128 rows, N = 128 columns, K = 64
              if (!(ok = mbar_wait_warp(FULL_T(st), (nJ >> 1) & 1, wc, W_MMA_FULL_J))) break;
              if (!(ok = mbar_wait_warp(S_EMPTY, (nt & 1) ^ 1, wc, W_MMA_S_EMPTY))) break;
              tc_fence_after();
              const uint32_t xtj = dXtJ_k0 + st * J_STEP, xsj = dXsJ_k0 + st * J_STEP;
#pragma unroll
              for (int k = 0; k < D / 16; ++k)
                umma_bf16_w_lead(lead, tmem + T_S, dXtR_k[rs] + k * 2, HI_1024, xtj + k * 2,
                                 HI_1024, IDESC_S, k > 0 ? 1u : 0u);
              issued = true;
              if (last_p) umma_commit_lead(lead, EMPTY_T(st));
              if (!(ok = mbar_wait_warp(FULL_S(st), (nJ >> 1) & 1, wc, W_MMA_FULL_J))) break;
              tc_fence_after();
#pragma unroll
              for (int k = 0; k < D / 16; ++k)
                umma_bf16_w_lead(lead, tmem + T_S + BN, dXsR_k[rs] + k * 2, HI_1024, xsj + k * 2,
                                 HI_1024, IDESC_S, k > 0 ? 1u : 0u);
              umma_commit_lead(lead, S_FULL);
            } else {
              // dX_R += G X_s[J] and P (+)= G^T X_s[R] for tile (R, J).  G_FULL
              // implies the tile's logits (hence its column tiles) are complete.
              const int pb = np & 1, gb = nt & 1;
              if (!(ok = mbar_wait_warp(G_FULL(gb), (nt >> 1) & 1, wc, W_MMA_G_FULL))) break;
              if (first_p && !(ok = mbar_wait_warp(P_EMPTY(pb), ((np >> 1) & 1) ^ 1, wc, W_MMA_P_EMPTY)))
                break;
              if (first_seq && !(ok = mbar_wait_warp(DXI_EMPTY, (nseq & 1) ^ 1, wc, W_MMA_DXI_EMPTY)))
                break;
              first_seq = false;
              tc_fence_after();
              const uint32_t xsj = dXsJ_mn0 + st * J_STEP;
              // M = i, N = c (64), K = j (128): G K-major steps 32 B in a row and a
              // box every 4 steps; X_s[J] MN-major steps 16 rows (2 KB)
#pragma unroll
              for (int k = 0; k < BN / 16; ++k)
                umma_bf16_w_lead(lead, tmem + T_DX0 + rs * D,
                                 dG_k + gb * G_STEP + (k >> 2) * BOX_STEP + (k & 3) * 2,
                                 HI_1024, xsj + k * 128, HI_1024, IDESC_GX, (J > 0 || k > 0) ? 1u : 0u);
              // M = j (128, two 64-column boxes of G, LBO = box), N = c (64), K = i (128)
#pragma unroll
              for (int k = 0; k < BM / 16; ++k)
                umma_bf16_w_lead(lead, tmem + T_P + pb * D, dG_mn + gb * G_STEP + k * 128, HI_1024,
                                 dXsR_mn[rs] + k * 128, HI_1024, IDESC_P,
                                 (!first_p || k > 0) ? 1u : 0u);
              issued = true;
              umma_commit_lead(lead, G_EMPTY(gb));
              if (last_p) {
                umma_commit_lead(lead, P_FULL(pb));
                umma_commit_lead(lead, EMPTY_S(st));
                ++np;
              }
            }
            ++nt;
          }
          ++nJ;
        }
        if (!ok) break;
        if (!is_logit) {
          umma_commit_lead(lead, EMPTY_I);
          umma_commit_lead(lead, DXI_FULL);
        }
        ++nseq;
      }
    }
    if (issued) {
      const uint32_t drain = is_logit ? DRAIN_L : DRAIN_G;
      umma_commit_lead(lead, drain);
      mbar_wait_drain(drain, 0, kDrainNs);
    }
    __syncwarp();
  } else if (warp >= BWD_EPI_WARP) {
    // ------------------------------------------------------- epilogue
    // Every f32 addition into dX goes out as a TMA reduce-add of a 32 x 32
    // box staged in this warp's 4 KB of shared memory (128-byte swizzle, one
    // 128-byte row per lane).  Lane 32q + l of P holds dX[J*128 + 32q + l][0:64].
    const int q = warp - BWD_EPI_WARP;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t stg = base + L::STG + q * L::STG_BYTES;
    const uint32_t rowp = stg + lane * 128;
    uint32_t np = 0, nseq = 0;
    bool ok = true;
    // stage 32 columns of this lane's row and add the box at (c0, row0)
    auto stage_add = [&](const float (&v)[32], const CUtensorMap* map, int c0, int row0, const Unit& U) {
      if (lane == 0) bulk_wait_read<0>();   // the previous box has left the buffer
      __syncwarp();
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4)
        st_shared_v4(rowp + ((k4 ^ (lane & 7)) << 4), __float_as_uint(v[4 * k4]),
                     __float_as_uint(v[4 * k4 + 1]), __float_as_uint(v[4 * k4 + 2]),
                     __float_as_uint(v[4 * k4 + 3]));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (row0 < p.N) tma_reduce_add_4d(map, stg, c0, row0, U.h, U.b);
        bulk_commit();
      }
    };
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      int u, m;
      decode_item(p, item, u, m);
      const Unit U = decode_unit(p, u);
      for (int w = 0; ok && w < 2; ++w) {
        const int R0 = pair_seq_block(U, m, w);
        if (R0 < 0) break;
        const bool has1 = R0 + 1 < U.nblk;
        const int nT = n_col_tiles_s<SYM>(p, U, has1 ? R0 + 1 : R0);
        for (int J = 0; J < nT; ++J) {
          const int b = np & 1;
          ok = mbar_wait(P_FULL(b), (np >> 1) & 1, wc, W_EPI_P_FULL);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int cb = 0; cb < D / 32; ++cb) {
            float v[32];
            tmem_ld32(tmem + lane_addr + T_P + b * D + cb * 32, v);
            tmem_wait_ld();
            if (cb == D / 32 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(P_EMPTY(b));
            }
            stage_add(v, &U.seg->tm_dx, cb * 32, U.tok0 + J * BN + q * 32, U);
          }
          ++np;
        }
        if (!ok) break;
        // dX rows of the pair: lane = row, 32-column boxes
        ok = mbar_wait(DXI_FULL, nseq & 1, wc, W_EPI_DXI_FULL);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        for (int rs = 0; rs < 2; ++rs) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float v[32];
            tmem_ld32(tmem + lane_addr + T_DX0 + rs * D + c * 32, v);
            tmem_wait_ld();
            if (rs == 1 && c == D / 32 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(DXI_EMPTY);
            }
            if (rs == 1 && !has1) continue;
            stage_add(v, &U.seg->tm_dx, c * 32, U.tok0 + (R0 + rs) * BM + q * 32, U);
          }
        }
        ++nseq;
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    // --------------------------------------------------- row warpgroups
    const int q = warp & 3;
    const int wg = warp >> 2;      // 32-column quarter of each 128-column tile
    const int r = q * 32 + lane;
    const float sl2 = p.sl2;
    // this thread's 64-byte slice of row r of G: box wg/2, chunks 4*(wg&1)..+3
    const uint32_t gsm0 = base + L::G + (wg >> 1) * L::TILE + r * 128;
    uint32_t nt = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
      int u, m;
      decode_item(p, item, u, m);
      const Unit U = decode_unit(p, u);
      for (int w = 0; ok && w < 2; ++w) {
        const int R0 = pair_seq_block(U, m, w);
        if (R0 < 0) break;
        const bool has1 = R0 + 1 < U.nblk;
        const int nT0 = n_col_tiles_s<SYM>(p, U, R0);
        const int nT = has1 ? n_col_tiles_s<SYM>(p, U, R0 + 1) : nT0;
        const int Lu = U.len;
        // per-row constants of both row blocks
        float bt[2], bs[2], mul[2];
        int lim[2];
#pragma unroll
        for (int rs = 0; rs < 2; ++rs) {
          const int row = (R0 + rs) * BM + r;
          const bool rvalid = row < Lu && (rs == 0 || has1);
          bt[rs] = bs[rs] = mul[rs] = 0.f;
          if (rvalid) {
            const float4 st4 = reinterpret_cast<const float4*>(U.seg->stats)[U.row0 + row];
            bt[rs] = -st4.y * kLog2e;
            bs[rs] = -st4.z * kLog2e;
            const float up = U.seg->dkl ? U.seg->dkl[U.row0 + row] : 1.0f / static_cast<float>(Lu);
            mul[rs] = up * p.scale;   // the logit scale of dX_s is folded into G
          }
          lim[rs] = !rvalid ? -1 : (p.causal ? min(row, Lu - 1) : Lu - 1);
          if (lim[rs] == 0) mul[rs] = 0.f;   // one allowed entry: R_t = R_s = 1, the gradient is 0
        }
        const float2 sl2v = make_float2(sl2, sl2), m1 = make_float2(-1.f, -1.f);
        for (int J = 0; ok && J < nT; ++J) {
          for (int rs = 0; rs < 2; ++rs) {
            if (rs == 0 && J >= nT0) continue;
            if (rs == 1 && !has1) continue;
            // full mask, off the diagonal tile: each lane fetches the partner
            // constants of one of this warpgroup's 32 columns while the logits
            // are still being computed
            const bool off = SYM && J < R0 + rs;
            PartnerCol pc{0.f, 0.f, 0.f};
            if (off) pc = partner_column(U, p, J * BN + wg * 32 + lane);
            ok = mbar_wait(S_FULL, nt & 1, wc, W_SM_S_FULL);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const uint32_t ta = tmem + (static_cast<uint32_t>(q * 32) << 16) + T_S + wg * 32;
            const float btr = rs ? bt[1] : bt[0], bsr = rs ? bs[1] : bs[0];
            const float mr = rs ? mul[1] : mul[0];
            const int limr = rs ? lim[1] : lim[0];
            const int col0 = J * BN + wg * 32;
            const uint32_t gsm = gsm0 + (nt & 1) * L::G_BYTES;
            if constexpr (SYM) {
              // full mask: 4 exps per entry off the diagonal tile, so the exps
              // bound this mode; the logits are read in two 16-column halves
              // (the second half releases the buffer), which keeps registers
              // free for the partners' shuffles
#pragma unroll 1
              for (int hf = 0; hf < 2; ++hf) {
                float t[16], s[16];
                tmem_ld16(ta + hf * 16, t);
                tmem_ld16(ta + BN + hf * 16, s);
                tmem_wait_ld();
                if (hf == 1) {
                  tc_fence_before();
                  __syncwarp();
                  if (lane == 0) mbar_arrive(S_EMPTY);
                } else {
                  // the gradient MMAs of two tiles back have read this G buffer
                  ok = mbar_wait(G_EMPTY(nt & 1), ((nt >> 1) & 1) ^ 1, wc, W_SM_G_EMPTY);
                  ok = __all_sync(0xffffffffu, ok);
                  if (!ok) break;
                }
                form_g_store<16>(t, s, btr, bsr, mr, col0 + hf * 16, limr, off, pc, hf * 16, p,
                                 gsm, (wg & 1) * 4 + hf * 2, r);
              }
              if (!ok) break;
            } else {
              // causal: read the whole slice of the tile at once and release the
              // logit buffer at once, so the next tile's logit MMAs overlap this
              // tile's exps (measured faster than two half loads despite the
              // register pressure)
              float t[32], s[32];
              tmem_ld32(ta, t);
              tmem_ld32(ta + BN, s);
              tmem_wait_ld();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(S_EMPTY);
              // the gradient MMAs of two tiles back have read this G buffer
              ok = mbar_wait(G_EMPTY(nt & 1), ((nt >> 1) & 1) ^ 1, wc, W_SM_G_EMPTY);
              ok = __all_sync(0xffffffffu, ok);
              if (!ok) break;
              form_g_store<32>(t, s, btr, bsr, mr, col0, limr, false, pc, 0, p, gsm,
                               (wg & 1) * 4, r);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(G_FULL(nt & 1));
            ++nt;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == BWDP_LOGIT_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------- schedule check (host)
// The kernels' work decomposition replayed on the host: every part's work
// items are decoded with the same helpers the kernels use, and the (unit,
// row block, column tile) triples they visit are compared with the triples the
// mask requires, worked out independently from row and column ranges: each
// must be visited exactly once over the parts, no other may be, and every
// visited tile's TMA row coordinates must lie inside the tensor.
namespace {
struct HostUnitSrc {
  const int* const* lens;
  const int* const* offs;
  // host copies; declared for both sides only because make_unit is
  __host__ __device__ int len(int r, int b) const { return lens[r][b]; }
  __host__ __device__ int cu(int r, int k) const { return offs[r][k]; }
};
}  // namespace

enum SchedKind { FWD, TC64, PAIR, PAIR64 };

static int schedule_check_kind(const TcParams& p0, SchedKind kind, int n_parts,
                               const int* const* lens, const int* const* offs, char* why,
                               size_t why_len) {
  const HostUnitSrc src{lens, offs};
  auto fail = [&](const char* what, int u, int R, int J) {
    if (why && why_len) snprintf(why, why_len, "%s (unit %d, row block %d, column tile %d)", what, u, R, J);
    return 1;
  };
  const int W = (kind == FWD || kind == PAIR64) ? 128 : 64;
  const bool tri = p0.causal || (kind == PAIR || kind == PAIR64);   // lower triangle only
  std::vector<std::vector<unsigned char>> seen(p0.n_units);
  std::vector<Unit> units(p0.n_units);
  for (int u = 0; u < p0.n_units; ++u) {
    units[u] = make_unit(p0, u, src);
    const int ncol = (units[u].span + W - 1) / W;
    seen[u].assign(static_cast<size_t>(units[u].nblk) * (ncol > 0 ? ncol : 1), 0);
  }
  auto visit = [&](int u, int R, int J) -> int {
    const Unit& U = units[u];
    const int ncol = (U.span + W - 1) / W;
    if (R < 0 || R >= U.nblk || J < 0 || J >= ncol) return fail("tile outside the unit", u, R, J);
    if (U.tok0 + R * BM >= p0.N || U.tok0 + J * W >= p0.N)
      return fail("TMA row coordinate outside the tensor", u, R, J);
    unsigned char& c = seen[u][static_cast<size_t>(R) * ncol + J];
    if (c) return fail("tile visited twice", u, R, J);
    c = 1;
    return 0;
  };
  for (int part = 0; part < n_parts; ++part) {
    TcParams p = p0;
    p.part = part;
    p.n_parts = n_parts;
    if (kind == PAIR || kind == PAIR64) p.n_pairs = ((p0.nblk + 1) / 2 + 1) / 2;
    p.n_local = part < p.n_pairs ? (p.n_pairs - part + n_parts - 1) / n_parts : 0;
    p.n_items = p.n_units * p.n_local;
    for (int item = 0; item < p.n_items; ++item) {
      int u, pp;
      decode_item(p, item, u, pp);
      if (u < 0 || u >= p.n_units) return fail("work item decodes to no unit", u, -1, -1);
      const Unit& U = units[u];
      if (kind == FWD || kind == TC64) {
        for (int pass = 0; pass < item_passes(U, pp); ++pass) {
          const int I = pass_block(U, pp, pass);
          const int nT = kind == FWD ? n_col_tiles(p, U, I) : n_col_tiles64(p, U, I);
          for (int J = 0; J < nT; ++J)
            if (visit(u, I, J)) return 1;
        }
      } else {
        for (int w = 0; w < 2; ++w) {
          const int R0 = pair_seq_block(U, pp, w);
          if (R0 < 0) break;
          for (int rs = 0; rs < 2 && R0 + rs < U.nblk; ++rs) {
            const int R = R0 + rs;
            const int nT = kind == PAIR64 ? (tri ? n_col_tiles_s<true>(p, U, R)
                                                 : n_col_tiles_s<false>(p, U, R))
                                          : (tri ? n_col_tiles64_s<true>(p, U, R)
                                                 : n_col_tiles64_s<false>(p, U, R));
            for (int J = 0; J < nT; ++J)
              if (visit(u, R, J)) return 1;
          }
        }
      }
    }
  }
  // every tile the mask needs: columns up to the block's last row (lower
  // triangle), or every column
  for (int u = 0; u < p0.n_units; ++u) {
    const Unit& U = units[u];
    const int ncol = (U.span + W - 1) / W;
    for (int R = 0; R < U.nblk; ++R) {
      const int need = tri ? imin((R * BM + BM + W - 1) / W, ncol) : ncol;
      for (int J = 0; J < ncol; ++J) {
        const bool got = seen[u][static_cast<size_t>(R) * ncol + J] != 0;
        if (J < need && !got) return fail("tile never visited", u, R, J);
        if (J >= need && got) return fail("tile outside the mask visited", u, R, J);
      }
    }
  }
  return 0;
}

int schedule_check(const TcParams& p0, int d, bool bwd, int n_parts, const int* const* lens,
                   const int* const* offs, char* why, size_t why_len) {
  // the kernels a launch of these shapes may run (the choice between the two
  // causal d = 128 backwards also depends on the SM count: both are checked)
  SchedKind kinds[2];
  int n = 0;
  if (!bwd) kinds[n++] = FWD;
  else if (d == 64) kinds[n++] = PAIR64;
  else if (!p0.causal || p0.nblk >= kPairAlwaysBlocks) kinds[n++] = PAIR;
  else if (p0.nblk < kPairMinBlocks) kinds[n++] = TC64;
  else {
    kinds[n++] = TC64;
    kinds[n++] = PAIR;
  }
  for (int i = 0; i < n; ++i)
    if (schedule_check_kind(p0, kinds[i], n_parts, lens, offs, why, why_len)) return 1;
  return 0;
}

// The paired-block kernels' work items for the part p describes: ceil(npb / 2)
// per unit, npb = ceil(nblk / 2), shared out like the one-block items.
static TcParams pair_schedule(const TcParams& p) {
  TcParams q = p;
  q.n_pairs = ((p.nblk + 1) / 2 + 1) / 2;
  q.n_local = q.part < q.n_pairs ? (q.n_pairs - q.part + q.n_parts - 1) / q.n_parts : 0;
  q.n_items = q.n_units * q.n_local;
  return q;
}

// Backward kernel of a tensor-core launch on `sms` SMs: 2 = one 128-row block
// per pass (relkl_bwd_tc64_kernel), 3 = adjacent row-block pairs
// (relkl_bwd_pair_kernel), 4 = pairs at d = 64 (relkl_bwd_pair64_kernel).
// Between 16 and 32 row blocks of a causal mask it compares estimated times:
// rounds of work items over the SMs times the item's length.  A paired item
// covers twice the tiles of a one-block item and runs them ~6 % faster
// (measured at 2K and 4K), so it costs 1.88 one-block items; the one-block
// kernel's finer items win where the paired kernel's last round would leave
// many SMs idle (few units: 96 units at N = 4096 run in 11 one-block rounds
// against 6 paired ones).
int tc_bwd_kind(const TcParams& p, int d, int sms) {
  if (d == 64) return 4;
  if (!p.causal || p.nblk >= kPairAlwaysBlocks) return 3;
  if (p.nblk < kPairMinBlocks || sms < 1) return 2;
  const long long one = p.n_items, pair = pair_schedule(p).n_items;
  const long long r1 = (one + sms - 1) / sms, r2 = (pair + sms - 1) / sms;
  return r2 * 188 < r1 * 100 ? 3 : 2;
}

// ------------------------------------------------------------ launchers
template <int D>
static cudaError_t launch_fwd(const TcParams& p, int grid, cudaStream_t stream) {
  auto k = relkl_fwd_tc_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       FwdSmem<D>::ALLOC);
  if (e != cudaSuccess) return e;
  k<<<grid, FWD_THREADS, FwdSmem<D>::ALLOC, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t tc_launch_fwd(const TcParams& p, int d, int grid, cudaStream_t stream) {
  return d == 64 ? launch_fwd<64>(p, grid, stream) : launch_fwd<128>(p, grid, stream);
}

// `max_grid`: the number of SMs; the grid is one CTA per SM or one per work
// item of the kernel chosen, whichever is fewer.
cudaError_t tc_launch_bwd(const TcParams& p, int d, int max_grid, cudaStream_t stream) {
  int grid = p.n_items < max_grid ? p.n_items : max_grid;
  const int kind = tc_bwd_kind(p, d, max_grid);
  if (kind == 4) {
    const TcParams q = pair_schedule(p);
    if (q.n_items == 0) return cudaSuccess;
    grid = q.n_items < max_grid ? q.n_items : max_grid;
    auto k = p.causal ? relkl_bwd_pair64_kernel<false> : relkl_bwd_pair64_kernel<true>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         BwdPair64Smem::ALLOC);
    if (e != cudaSuccess) return e;
    k<<<grid, BWDP_THREADS, BwdPair64Smem::ALLOC, stream>>>(q);
    return cudaGetLastError();
  }
  // full masks take the paired-block kernel at every N (it serves both
  // orientations of each off-diagonal tile); causal ones with few row blocks
  // may take the one-block kernel, whose finer work items balance better
  if (kind == 2) {
    if (!grid) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(relkl_bwd_tc64_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Bwd64Smem::ALLOC);
    if (e != cudaSuccess) return e;
    relkl_bwd_tc64_kernel<<<grid, BWD_THREADS, Bwd64Smem::ALLOC, stream>>>(p);
    return cudaGetLastError();
  }
  const TcParams q = pair_schedule(p);
  if (q.n_items == 0) return cudaSuccess;
  grid = q.n_items < max_grid ? q.n_items : max_grid;
  auto k = p.causal ? relkl_bwd_pair_kernel<false> : relkl_bwd_pair_kernel<true>;
  const int alloc = p.causal ? BwdPairSmem<false>::ALLOC : BwdPairSmem<true>::ALLOC;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, alloc);
  if (e != cudaSuccess) return e;
  k<<<grid, BWDP_THREADS, alloc, stream>>>(q);
  return cudaGetLastError();
}


}  // namespace relkl
