// Kernel parameter blocks shared by the launch code and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace relkl {

struct DevStatus;

constexpr int kMaxSeg = 3;   // relations per launch (Q, K, V)

// One relation inside a launch.  Units of relation r are numbered
// unit_begin .. unit_begin + B*H - 1, batch-major then head.
struct TcSeg {
  CUtensorMap tm_t;          // teacher [B,H,N,d] bf16, box 64 cols x 128 rows, 128B swizzle
  CUtensorMap tm_s;          // student, same geometry
  CUtensorMap tm_dx;         // dX [B,H,N,d] f32, box 32 cols x 32 rows, 128B swizzle (bwd)
  CUtensorMap tm_t64;        // teacher, box 64 cols x 64 rows (bwd column tiles, d = 128)
  CUtensorMap tm_s64;        // student, same geometry
  float* kl;                 // [B,H,N]
  float* stats;              // [B,H,N,4]
  const float* dkl;          // [B,H,N] or null (1/N)
  float* dx;                 // [B,H,N,d] float32
  const int* lengths;        // [B] valid lengths (device) or null (all N)
  const int* cu_seqlens;     // packed sequences: [n_seq + 1] token offsets (device), or null
  int B, H;                  // packed sequences: B = n_seq (units are (sequence, head))
  int unit_begin;
  int max_seqlen;            // packed sequences: bound on every sequence's length
};

struct TcParams {
  TcSeg seg[kMaxSeg];
  int n_seg;
  int N;
  int nblk;       // ceil(N / 128)
  int n_pairs;    // work items per unit (forward: ceil(nblk / 2), row blocks p and nblk-1-p)
  int n_units;
  // A call may cover one part of every unit's work items: items
  // part, part + n_parts, ... (rows of the other parts are not touched).
  int part, n_parts;
  int n_local;    // items per unit in this part: ceil((n_pairs - part) / n_parts)
  int n_items;    // n_units * n_local
  int causal;
  float scale;    // logit scale
  float sl2;      // scale * log2(e)
  DevStatus* status;
  unsigned long long timeout_ns;
};

// CUDA-core float32 path: plain pointers with element strides.
struct SimtSeg {
  const void* xt;
  const void* xs;
  int64_t sb, sh, sn;        // element strides of B, H, N (d is contiguous)
  float* kl;
  float* stats;
  const float* dkl;
  float* dx;
  const int* lengths;        // [B] valid lengths (device) or null (all N)
  const int* cu_seqlens;     // packed sequences: [n_seq + 1] token offsets, or null
  int B, H;                  // packed sequences: B = n_seq
  int unit_begin;
  int max_seqlen;
};

struct SimtParams {
  SimtSeg seg[kMaxSeg];
  int n_seg;
  int N, d;
  int causal;
  int is_bf16;
  float scale;
  int n_units;
  int part, n_parts;   // 32-row blocks part, part + n_parts, ... of every unit
  int nblk_local;      // ceil((ceil(N / 32) - part) / n_parts)
};

}  // namespace relkl
