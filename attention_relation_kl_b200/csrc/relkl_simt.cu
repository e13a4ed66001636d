// CUDA-core float32 kernels for the relation KL (any head dim 1..128, fp32 or
// bf16 inputs).  They compute the same quantities as the tensor-core path --
// LinearARD's per-row forward KL of the masked row-softmaxed self-relations
// and dX_s = s (G + G^T) X_s with G = dkl (R_s - R_t) (pith.science verdict,
// pith_extraction.key_machinery) -- with plain fp32 FMAs and accurate expf /
// logf, one 32-row block per CTA and 32-column tiles.  They serve the fp32
// workloads, where no tensor-core rounding is wanted, and head dims the
// tensor-core kernels do not cover.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "relkl_params.h"

namespace relkl {

constexpr int SB = 32;           // rows per block and columns per tile
constexpr int SIMT_THREADS = 256;  // 32 rows x 8 column groups of 4

__device__ __forceinline__ float load_x(const void* base, int is_bf16, int64_t off) {
  if (is_bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[off]);
  return reinterpret_cast<const float*>(base)[off];
}

struct SimtUnit {
  const SimtSeg* seg;
  int64_t xoff;   // element offset of the unit's first row in x
  int64_t row0;   // first row of the unit in [B,H,N] arrays
  int L;          // valid rows and columns (its batch element's length, or N)
  int span;       // rows the unit covers: its length for a packed sequence, else N
};

// Unit u: (b, h) of a batched relation, or (sequence k, head h) of packed
// sequences (sequence k on tokens [cu_seqlens[k], cu_seqlens[k+1]) of [1,H,N,d]).
__device__ __forceinline__ SimtUnit simt_unit(const SimtParams& p, int u) {
  int r = 0;
  for (int k = 1; k < p.n_seg; ++k)
    if (u >= p.seg[k].unit_begin) r = k;
  const SimtSeg* s = &p.seg[r];
  const int local = u - s->unit_begin;
  const int b = local / s->H, h = local - (local / s->H) * s->H;
  SimtUnit out;
  out.seg = s;
  if (s->cu_seqlens) {
    const int a = min(max(s->cu_seqlens[b], 0), p.N);
    const int e = min(max(s->cu_seqlens[b + 1], a), p.N);
    out.L = min(e - a, s->max_seqlen);
    out.span = out.L;
    out.xoff = h * s->sh + a * s->sn;
    out.row0 = static_cast<int64_t>(h) * p.N + a;
  } else {
    out.L = s->lengths ? max(0, min(p.N, s->lengths[b])) : p.N;   // valid rows and columns
    out.span = p.N;
    out.xoff = b * s->sb + h * s->sh;
    out.row0 = (static_cast<int64_t>(b) * s->H + h) * p.N;
  }
  return out;
}

// Stage rows [r0, r0+32) of x (teacher or student) into shared memory with a
// row pitch of d+1 floats; rows past N are zero.
__device__ __forceinline__ void stage_rows(float* dst, const void* x, int is_bf16, int64_t xoff,
                                           int64_t sn, int r0, int N, int d) {
  for (int e = threadIdx.x; e < SB * d; e += blockDim.x) {
    const int rr = e / d, k = e - (e / d) * d;
    const int row = r0 + rr;
    dst[rr * (d + 1) + k] = row < N ? load_x(x, is_bf16, xoff + row * sn + k) : 0.f;
  }
}

__global__ void __launch_bounds__(SIMT_THREADS)
relkl_fwd_simt_kernel(const __grid_constant__ SimtParams p) {
  extern __shared__ float sm[];
  const int d = p.d, pitch = d + 1;
  float* xti = sm;
  float* xsi = xti + SB * pitch;
  float* xtj = xsi + SB * pitch;
  float* xsj = xtj + SB * pitch;

  // this call's 32-row blocks of the unit: part, part + n_parts, ...
  const int u = blockIdx.x / p.nblk_local;
  const int I = p.part + (blockIdx.x - u * p.nblk_local) * p.n_parts;
  const SimtUnit U = simt_unit(p, u);
  const SimtSeg& S = *U.seg;
  const int rr = threadIdx.x >> 3, cg = threadIdx.x & 7;
  const int row = I * SB + rr;
  const float sc = p.scale;

  if (I * SB >= U.span) return;   // a block past a short packed sequence
  stage_rows(xti, S.xt, p.is_bf16, U.xoff, S.sn, I * SB, U.span, d);
  stage_rows(xsi, S.xs, p.is_bf16, U.xoff, S.sn, I * SB, U.span, d);

  float m_run = -INFINITY, St = 0.f, C = 0.f, A = 0.f;
  const int nJ = p.causal ? I + 1 : (U.span + SB - 1) / SB;
  for (int J = 0; J < nJ; ++J) {
    __syncthreads();
    stage_rows(xtj, S.xt, p.is_bf16, U.xoff, S.sn, J * SB, U.span, d);
    stage_rows(xsj, S.xs, p.is_bf16, U.xoff, S.sn, J * SB, U.span, d);
    __syncthreads();
    float zt[4], zs[4];
    bool ok[4];
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int jj = cg * 4 + c, col = J * SB + jj;
      float at = 0.f, as = 0.f;
      for (int k = 0; k < d; ++k) {
        at = fmaf(xti[rr * pitch + k], xtj[jj * pitch + k], at);
        as = fmaf(xsi[rr * pitch + k], xsj[jj * pitch + k], as);
      }
      zt[c] = at * sc;
      zs[c] = as * sc;
      ok[c] = row < U.L && col < U.L && (!p.causal || col <= row);
      if (ok[c]) mx = fmaxf(mx, fmaxf(zt[c], zs[c]));
    }
    // the 8 lanes of a row share one running maximum
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (mx > m_run) {
      const float a = expf(m_run - mx);
      St *= a;
      C *= a;
      A *= a;
      m_run = mx;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (!ok[c]) continue;
      const float et = expf(zt[c] - m_run), es = expf(zs[c] - m_run);
      St += et;
      C += es - et;
      A = fmaf(et, zt[c] - zs[c], A);
    }
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    St += __shfl_xor_sync(0xffffffffu, St, o);
    C += __shfl_xor_sync(0xffffffffu, C, o);
    A += __shfl_xor_sync(0xffffffffu, A, o);
  }
  if (cg == 0 && row < U.span && row >= U.L) {   // padding row
    S.kl[U.row0 + row] = 0.f;
    reinterpret_cast<float4*>(S.stats)[U.row0 + row] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else if (cg == 0 && row < U.span) {
    const float lse_t = m_run + logf(St);
    const float l1 = log1pf(C / St);
    const float w = A / St;
    const int64_t g = U.row0 + row;
    S.kl[g] = w + l1;
    reinterpret_cast<float4*>(S.stats)[g] = make_float4(m_run, lse_t, lse_t + l1, w);
  }
}

__global__ void __launch_bounds__(SIMT_THREADS)
relkl_bwd_simt_kernel(const __grid_constant__ SimtParams p) {
  extern __shared__ float sm[];
  const int d = p.d, pitch = d + 1;
  float* xti = sm;
  float* xsi = xti + SB * pitch;
  float* xtj = xsi + SB * pitch;
  float* xsj = xtj + SB * pitch;
  float* g = xsj + SB * pitch;      // [32][33]

  // this call's 32-row blocks of the unit: part, part + n_parts, ...
  const int u = blockIdx.x / p.nblk_local;
  const int I = p.part + (blockIdx.x - u * p.nblk_local) * p.n_parts;
  const SimtUnit U = simt_unit(p, u);
  const SimtSeg& S = *U.seg;
  const int rr = threadIdx.x >> 3, cg = threadIdx.x & 7;
  const int row = I * SB + rr;
  const float sc = p.scale;

  if (I * SB >= U.span) return;   // a block past a short packed sequence
  stage_rows(xti, S.xt, p.is_bf16, U.xoff, S.sn, I * SB, U.span, d);
  stage_rows(xsi, S.xs, p.is_bf16, U.xoff, S.sn, I * SB, U.span, d);
  float lse_t = 0.f, lse_s = 0.f, mul = 0.f;
  if (row < U.L) {
    const float4 st4 = reinterpret_cast<const float4*>(S.stats)[U.row0 + row];
    lse_t = st4.y;
    lse_s = st4.z;
    mul = (S.dkl ? S.dkl[U.row0 + row] : 1.0f / static_cast<float>(U.L)) * sc;
    // a row with one allowed entry has R_t = R_s = 1 there: its gradient is
    // exactly zero (left to the exps, float32 rounding of logits and LSEs of
    // size ~|z| would leave ~|z| 2^-24 of it, times the row's upstream weight)
    if (p.causal ? row == 0 : U.L == 1) mul = 0.f;
  }
  // dX_I accumulator: this thread owns columns cg, cg+8, ... of row rr
  constexpr int MAXC = 128 / 8;
  float acc[MAXC];
#pragma unroll
  for (int m = 0; m < MAXC; ++m) acc[m] = 0.f;

  const int nJ = p.causal ? I + 1 : (U.span + SB - 1) / SB;
  for (int J = 0; J < nJ; ++J) {
    __syncthreads();
    stage_rows(xtj, S.xt, p.is_bf16, U.xoff, S.sn, J * SB, U.span, d);
    stage_rows(xsj, S.xs, p.is_bf16, U.xoff, S.sn, J * SB, U.span, d);
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int jj = cg * 4 + c, col = J * SB + jj;
      float at = 0.f, as = 0.f;
      for (int k = 0; k < d; ++k) {
        at = fmaf(xti[rr * pitch + k], xtj[jj * pitch + k], at);
        as = fmaf(xsi[rr * pitch + k], xsj[jj * pitch + k], as);
      }
      const bool ok = row < U.L && col < U.L && (!p.causal || col <= row);
      g[rr * (SB + 1) + jj] = ok ? mul * (expf(as * sc - lse_s) - expf(at * sc - lse_t)) : 0.f;
    }
    __syncthreads();
    // dX_I += G X_s[J]
#pragma unroll
    for (int m = 0; m < MAXC; ++m) {
      const int k = cg + 8 * m;
      if (k < d) {
        float a = acc[m];
        for (int jj = 0; jj < SB; ++jj) a = fmaf(g[rr * (SB + 1) + jj], xsj[jj * pitch + k], a);
        acc[m] = a;
      }
    }
    // dX[J] += G^T X_s[I]   (thread: column-block row jj = rr)
    const int jrow = J * SB + rr;
    if (jrow < U.span) {
      float* dst = S.dx + (U.row0 + jrow) * d;
      for (int k = cg; k < d; k += 8) {
        float a = 0.f;
        for (int ii = 0; ii < SB; ++ii) a = fmaf(g[ii * (SB + 1) + rr], xsi[ii * pitch + k], a);
        atomicAdd(dst + k, a);
      }
    }
  }
  if (row < U.span) {
    float* dst = S.dx + (U.row0 + row) * d;
#pragma unroll
    for (int m = 0; m < MAXC; ++m) {
      const int k = cg + 8 * m;
      if (k < d) atomicAdd(dst + k, acc[m]);
    }
  }
}

__global__ void relkl_zero_kernel(float4* __restrict__ p, int64_t n4) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

__global__ void relkl_zero_tail_kernel(float* __restrict__ p, int64_t n) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i < n) p[i] = 0.f;
}

static size_t simt_smem(int d, int bwd) {
  return (4 * SB * (d + 1) + (bwd ? SB * (SB + 1) : 0)) * sizeof(float);
}

cudaError_t simt_launch_fwd(const SimtParams& p, cudaStream_t stream) {
  if (p.n_units * p.nblk_local == 0) return cudaSuccess;
  const size_t sm = simt_smem(p.d, 0);
  cudaError_t e = cudaFuncSetAttribute(relkl_fwd_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sm));
  if (e != cudaSuccess) return e;
  relkl_fwd_simt_kernel<<<p.n_units * p.nblk_local, SIMT_THREADS, sm, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t simt_launch_bwd(const SimtParams& p, cudaStream_t stream) {
  if (p.n_units * p.nblk_local == 0) return cudaSuccess;
  const size_t sm = simt_smem(p.d, 1);
  cudaError_t e = cudaFuncSetAttribute(relkl_bwd_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sm));
  if (e != cudaSuccess) return e;
  relkl_bwd_simt_kernel<<<p.n_units * p.nblk_local, SIMT_THREADS, sm, stream>>>(p);
  return cudaGetLastError();
}

// Zero a float32 buffer of n elements (16-byte aligned base).
cudaError_t launch_zero(float* ptr, int64_t n, int num_sms, cudaStream_t stream) {
  const int64_t n4 = n / 4;
  if (n4 > 0) {
    int64_t blocks = (n4 + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    relkl_zero_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
        reinterpret_cast<float4*>(ptr), n4);
  }
  const int64_t tail = n - n4 * 4;
  if (tail > 0) relkl_zero_tail_kernel<<<1, 32, 0, stream>>>(ptr + n4 * 4, tail);
  return cudaGetLastError();
}

// ------------------------------------------------ bf16 copy of dX_s
// Round to nearest, ties to even (cvt.rn), eight elements per thread step:
// two 16-byte loads, one 16-byte store.  HBM-bound: 6 bytes per element.
__global__ void relkl_cast_bf16_kernel(const float4* __restrict__ src, uint4* __restrict__ dst,
                                       int64_t n8) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = src[2 * i], b = src[2 * i + 1];
    const __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
    const __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
    uint4 o;
    o.x = *reinterpret_cast<const uint32_t*>(&p0);
    o.y = *reinterpret_cast<const uint32_t*>(&p1);
    o.z = *reinterpret_cast<const uint32_t*>(&p2);
    o.w = *reinterpret_cast<const uint32_t*>(&p3);
    dst[i] = o;
  }
}

// Element by element: the ragged tail, or arrays not 16-byte aligned.
__global__ void relkl_cast_bf16_scalar_kernel(const float* __restrict__ src,
                                              __nv_bfloat16* __restrict__ dst, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

cudaError_t launch_cast_bf16(const float* src, void* dst, int64_t n, int num_sms,
                             cudaStream_t stream) {
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  auto blocks_for = [&](int64_t work) {
    const int64_t b = (work + 255) / 256;
    return static_cast<int>(b < cap ? b : cap);
  };
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(dst);
  const bool vec = (reinterpret_cast<uintptr_t>(src) % 16 == 0) &&
                   (reinterpret_cast<uintptr_t>(dst) % 16 == 0);
  const int64_t n8 = vec ? n / 8 : 0;
  if (n8 > 0)
    relkl_cast_bf16_kernel<<<blocks_for(n8), 256, 0, stream>>>(
        reinterpret_cast<const float4*>(src), reinterpret_cast<uint4*>(out), n8);
  const int64_t rest = n - n8 * 8;
  if (rest > 0)
    relkl_cast_bf16_scalar_kernel<<<blocks_for(rest), 256, 0, stream>>>(src + n8 * 8, out + n8 * 8,
                                                                        rest);
  return cudaGetLastError();
}

}  // namespace relkl
