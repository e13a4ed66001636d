// Host side of the C ABI declared in include/relkl.h: argument validation,
// TMA descriptor encoding, kernel selection and launch.  No allocation and no
// state survives a call except two process-wide settings (the wait timeout
// and a per-device SM-count cache).
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/relkl.h"
#include "relkl_device.cuh"
#include "relkl_params.h"

namespace relkl {
cudaError_t tc_launch_fwd(const TcParams& p, int d, int grid, cudaStream_t stream);
cudaError_t tc_launch_bwd(const TcParams& p, int d, int grid, cudaStream_t stream);
cudaError_t simt_launch_fwd(const SimtParams& p, cudaStream_t stream);
cudaError_t simt_launch_bwd(const SimtParams& p, cudaStream_t stream);
cudaError_t launch_zero(float* ptr, int64_t n, int num_sms, cudaStream_t stream);
cudaError_t launch_cast_bf16(const float* src, void* dst, int64_t n, int num_sms,
                             cudaStream_t stream);
int schedule_check(const TcParams& p0, int d, bool bwd, int n_parts, const int* const* lens,
                   const int* const* offs, char* why, size_t why_len);
int tc_bwd_kind(const TcParams& p, int d, int sms);
cudaError_t launch_rope_bwd(const float* dx, void* out, int B, int H, int N, int d, bool bf16_out,
                            double base, double pos_scale, double pos_offset, int apply,
                            cudaStream_t stream);
using EncodeTiledFnG = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
int launch_wgrad(EncodeTiledFnG encode, long long rows, int D, int cols, const void* h,
                 const void* dx_pre, float* dw, int num_sms, DevStatus* status,
                 unsigned long long timeout_ns, cudaStream_t stream);
}  // namespace relkl

using namespace relkl;

namespace {

constexpr size_t kWorkspaceBytes = 256;
std::atomic<unsigned long long> g_timeout_ns{2000000000ull};
thread_local int32_t g_last_cuda = 0;

relkl_status cuda_fail(cudaError_t e) {
  g_last_cuda = static_cast<int32_t>(e);
  return RELKL_ERR_CUDA;
}

// NVTX range over the host side of one entry point (validation, descriptor
// encoding, launches), so that a profiler timeline shows which call queued
// which kernels.  NVTX3 is header-only: without an attached tool the push and
// pop are a load and a branch.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// cuTensorMapEncodeTiled, fetched from the driver through the runtime so the
// library needs no link-time dependency on libcuda.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

EncodeTiledFn encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

struct DevInfo {
  int sms = 0;
  int major = 0;
};
DevInfo g_dev[64];
std::mutex g_dev_mu;

relkl_status device_info(DevInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return RELKL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_dev[dev].sms == 0) {
    int sms = 0, major = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) !=
        cudaSuccess)
      return cuda_fail(e);
    g_dev[dev].sms = sms;
    g_dev[dev].major = major;
  }
  *out = g_dev[dev];
  return RELKL_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Units of a desc: (b, h) of its [B, H, N, d] tensors, or (sequence, head)
// of packed sequences.
int64_t n_units(const relkl_desc& d) {
  return static_cast<int64_t>(d.cu_seqlens ? d.n_seq : d.B) * d.H;
}

relkl_status check_desc(const relkl_desc* d) {
  if (!d) return RELKL_ERR_INVALID;
  if (d->B < 0 || d->H < 0 || d->N < 0 || d->d < 1) return RELKL_ERR_INVALID;
  if (d->dtype != RELKL_BF16 && d->dtype != RELKL_FP32) return RELKL_ERR_INVALID;
  if (d->causal != 0 && d->causal != 1) return RELKL_ERR_INVALID;
  if (d->reserved != 0) return RELKL_ERR_INVALID;
  if (d->lengths && !aligned(d->lengths, 4)) return RELKL_ERR_INVALID;
  if (d->cu_seqlens) {
    if (!aligned(d->cu_seqlens, 4) || d->lengths || d->B != 1 || d->n_seq < 0 ||
        d->max_seqlen < 0 || d->max_seqlen > d->N)
      return RELKL_ERR_INVALID;
  } else if (d->n_seq != 0 || d->max_seqlen != 0) {
    return RELKL_ERR_INVALID;
  }
  if (!(d->scale >= 0.f) || !std::isfinite(d->scale)) return RELKL_ERR_INVALID;
  if (d->stride[3] != 1) return RELKL_ERR_INVALID;
  for (int i = 0; i < 3; ++i)
    if (d->stride[i] < 0) return RELKL_ERR_INVALID;
  if (d->d > 128) return RELKL_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->N) * d->d >= (int64_t(1) << 31)) return RELKL_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->B) * d->H * d->N >= (int64_t(1) << 40)) return RELKL_ERR_UNSUPPORTED;
  return RELKL_OK;
}

bool tc_shape(const relkl_desc& d) {
  return d.dtype == RELKL_BF16 && (d.d == 64 || d.d == 128);
}

// Tensor-core path needs 16-byte aligned bases and strides (TMA).
bool tc_layout_ok(const relkl_desc& d, const void* xt, const void* xs) {
  if (!aligned(xt, 16) || !aligned(xs, 16)) return false;
  for (int i = 0; i < 3; ++i)
    if ((d.stride[i] * 2) % 16 != 0) return false;
  return true;
}

float logit_scale(const relkl_desc& d) {
  return d.scale > 0.f ? d.scale : 1.0f / std::sqrt(static_cast<float>(d.d));
}

relkl_status encode_x(CUtensorMap* m, const relkl_desc& d, const void* x, cuuint32_t box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return RELKL_ERR_CUDA;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d.d), static_cast<cuuint64_t>(d.N),
                              static_cast<cuuint64_t>(d.H), static_cast<cuuint64_t>(d.B)};
  // a dimension of extent 1 may carry any stride; give it a legal one
  auto stride_or = [&](int i, int64_t fallback) {
    return static_cast<cuuint64_t>((d.stride[i] > 0 ? d.stride[i] : fallback) * 2);
  };
  const int64_t row = d.stride[2] > 0 ? d.stride[2] : d.d;
  const cuuint64_t strides[3] = {stride_or(2, d.d), stride_or(1, row * d.N),
                                 stride_or(0, row * d.N * d.H)};
  const cuuint32_t box[4] = {64, box_rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RELKL_OK : RELKL_ERR_UNSUPPORTED;
}

// dX [B,H,N,d] f32 contiguous: 4-D map, box 32 cols x 32 rows, 128B swizzle,
// the target of the backward's TMA reduce-adds.
relkl_status encode_dx(CUtensorMap* m, const relkl_desc& d, float* dx) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return RELKL_ERR_CUDA;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d.d), static_cast<cuuint64_t>(d.N),
                              static_cast<cuuint64_t>(d.H), static_cast<cuuint64_t>(d.B)};
  const cuuint64_t row = static_cast<cuuint64_t>(d.d) * 4;
  const cuuint64_t strides[3] = {row, row * d.N, row * d.N * d.H};
  const cuuint32_t box[4] = {32, 32, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dx, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RELKL_OK : RELKL_ERR_UNSUPPORTED;
}

relkl_status check_ws(const void* ws, size_t ws_bytes) {
  if (!ws || ws_bytes < kWorkspaceBytes || !aligned(ws, 256)) return RELKL_ERR_WORKSPACE;
  return RELKL_OK;
}

// Common validation of a multi-relation call.  Sets *empty when there is no
// work at all.
relkl_status check_multi(int32_t n_rel, const relkl_desc* descs, const void* const* xt,
                         const void* const* xs, bool* empty) {
  if (n_rel < 1 || n_rel > kMaxSeg || !descs || !xt || !xs) return RELKL_ERR_INVALID;
  int64_t units = 0;
  for (int r = 0; r < n_rel; ++r) {
    relkl_status s = check_desc(&descs[r]);
    if (s != RELKL_OK) return s;
    const relkl_desc& a = descs[0];
    const relkl_desc& b = descs[r];
    if (a.N != b.N || a.d != b.d || a.dtype != b.dtype || a.causal != b.causal ||
        a.scale != b.scale || (a.cu_seqlens == nullptr) != (b.cu_seqlens == nullptr) ||
        a.max_seqlen != b.max_seqlen)
      return RELKL_ERR_INVALID;
    units += n_units(b);
  }
  if (units >= (int64_t(1) << 30)) return RELKL_ERR_UNSUPPORTED;
  *empty = (units == 0 || descs[0].N == 0 || (descs[0].cu_seqlens && descs[0].max_seqlen == 0));
  if (*empty) return RELKL_OK;
  for (int r = 0; r < n_rel; ++r) {
    if (n_units(descs[r]) == 0) continue;
    if (!xt[r] || !xs[r]) return RELKL_ERR_INVALID;
    const size_t es = descs[r].dtype == RELKL_BF16 ? 2 : 4;
    if (!aligned(xt[r], es) || !aligned(xs[r], es)) return RELKL_ERR_INVALID;
  }
  return RELKL_OK;
}

bool use_tc(int32_t n_rel, const relkl_desc* descs, const void* const* xt, const void* const* xs) {
  if (!tc_shape(descs[0])) return false;
  for (int r = 0; r < n_rel; ++r)
    if (n_units(descs[r]) && !tc_layout_ok(descs[r], xt[r], xs[r])) return false;
  return true;
}

// The schedule fields of a tensor-core launch (everything but the tensor
// maps and pointers): shared by the launch and the host schedule check.
void fill_schedule(int32_t n_rel, const relkl_desc* descs, TcParams* p, int part, int n_parts) {
  std::memset(p, 0, sizeof(*p));
  const relkl_desc& d0 = descs[0];
  int seg = 0, ub = 0;
  for (int r = 0; r < n_rel; ++r) {
    if (n_units(descs[r]) == 0) continue;
    TcSeg& s = p->seg[seg];
    s.B = descs[r].cu_seqlens ? descs[r].n_seq : descs[r].B;
    s.H = descs[r].H;
    s.lengths = descs[r].lengths;
    s.cu_seqlens = descs[r].cu_seqlens;
    s.max_seqlen = descs[r].max_seqlen;
    s.unit_begin = ub;
    ub += static_cast<int>(n_units(descs[r]));
    ++seg;
  }
  p->n_seg = seg;
  p->N = d0.N;
  // rows a unit's work covers: every row, or at most max_seqlen of a packed sequence
  const int span = d0.cu_seqlens ? d0.max_seqlen : d0.N;
  p->nblk = (span + 127) / 128;
  p->n_pairs = (p->nblk + 1) / 2;
  p->n_units = ub;
  p->part = part;
  p->n_parts = n_parts;
  p->n_local = part < p->n_pairs ? (p->n_pairs - part + n_parts - 1) / n_parts : 0;
  p->n_items = ub * p->n_local;
  p->causal = d0.causal;
  p->scale = logit_scale(d0);
  p->sl2 = p->scale * 1.4426950408889634f;
}

relkl_status build_tc(int32_t n_rel, const relkl_desc* descs, const void* const* xt,
                      const void* const* xs, TcParams* p, void* ws, int part = 0,
                      int n_parts = 1) {
  fill_schedule(n_rel, descs, p, part, n_parts);
  for (int r = 0, seg = 0; r < n_rel; ++r) {
    if (n_units(descs[r]) == 0) continue;
    TcSeg& s = p->seg[seg++];
    relkl_status st = encode_x(&s.tm_t, descs[r], xt[r]);
    if (st != RELKL_OK) return st;
    if ((st = encode_x(&s.tm_s, descs[r], xs[r])) != RELKL_OK) return st;
  }
  p->status = reinterpret_cast<DevStatus*>(ws);
  p->timeout_ns = g_timeout_ns.load();
  return RELKL_OK;
}

relkl_status build_simt(int32_t n_rel, const relkl_desc* descs, const void* const* xt,
                        const void* const* xs, SimtParams* p, int part = 0, int n_parts = 1) {
  std::memset(p, 0, sizeof(*p));
  const relkl_desc& d0 = descs[0];
  int seg = 0, ub = 0;
  for (int r = 0; r < n_rel; ++r) {
    if (n_units(descs[r]) == 0) continue;
    SimtSeg& s = p->seg[seg];
    s.xt = xt[r];
    s.xs = xs[r];
    s.sb = descs[r].stride[0];
    s.sh = descs[r].stride[1];
    s.sn = descs[r].stride[2];
    s.B = descs[r].cu_seqlens ? descs[r].n_seq : descs[r].B;
    s.H = descs[r].H;
    s.lengths = descs[r].lengths;
    s.cu_seqlens = descs[r].cu_seqlens;
    s.max_seqlen = descs[r].max_seqlen;
    s.unit_begin = ub;
    ub += static_cast<int>(n_units(descs[r]));
    ++seg;
  }
  p->n_seg = seg;
  p->N = d0.N;
  p->d = d0.d;
  p->causal = d0.causal;
  p->is_bf16 = d0.dtype == RELKL_BF16;
  p->scale = logit_scale(d0);
  p->n_units = ub;
  p->part = part;
  p->n_parts = n_parts;
  const int nblk32 = ((d0.cu_seqlens ? d0.max_seqlen : d0.N) + 31) / 32;
  p->nblk_local = part < nblk32 ? (nblk32 - part + n_parts - 1) / n_parts : 0;
  return RELKL_OK;
}

// Index of relation r's segment (relations without units have none).
template <class P>
void set_seg_outputs(P* p, int32_t n_rel, const relkl_desc* descs, float* const* kl,
                     float* const* stats, const float* const* stats_in, const float* const* dkl,
                     float* const* dx) {
  int seg = 0;
  for (int r = 0; r < n_rel; ++r) {
    if (n_units(descs[r]) == 0) continue;
    auto& s = p->seg[seg++];
    if (kl) s.kl = kl[r];
    if (stats) s.stats = stats[r];
    if (stats_in) s.stats = const_cast<float*>(stats_in[r]);
    s.dkl = dkl ? dkl[r] : nullptr;
    if (dx) s.dx = dx[r];
  }
}

}  // namespace

extern "C" {

size_t relkl_workspace_bytes(void) { return kWorkspaceBytes; }

relkl_status relkl_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  relkl_status s = check_ws(ws, ws_bytes);
  if (s != RELKL_OK) return s;
  cudaError_t e = cudaMemsetAsync(ws, 0, kWorkspaceBytes, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RELKL_OK : cuda_fail(e);
}

int32_t relkl_path_for(const relkl_desc* desc) {
  if (check_desc(desc) != RELKL_OK) return 0;
  return tc_shape(*desc) ? 1 : 2;
}

}  // extern "C"

namespace {

#ifdef RELKL_CHECKS
// Debug builds (-DRELKL_CHECKS): replay the launch's schedule on the host
// before enqueueing it (synchronous copies of lengths / packed offsets).
relkl_status debug_schedule_check(int32_t n_rel, const relkl_desc* descs, bool bwd, int part,
                                  int n_parts) {
  std::vector<std::vector<int32_t>> lens(n_rel), offs(n_rel);
  const int32_t* lp[kMaxSeg] = {nullptr, nullptr, nullptr};
  const int32_t* op[kMaxSeg] = {nullptr, nullptr, nullptr};
  for (int r = 0; r < n_rel; ++r) {
    if (descs[r].lengths) {
      lens[r].resize(descs[r].B);
      if (cudaMemcpy(lens[r].data(), descs[r].lengths, 4 * descs[r].B, cudaMemcpyDeviceToHost) !=
          cudaSuccess)
        return RELKL_ERR_CUDA;
      lp[r] = lens[r].data();
    }
    if (descs[r].cu_seqlens) {
      offs[r].resize(descs[r].n_seq + 1);
      if (cudaMemcpy(offs[r].data(), descs[r].cu_seqlens, 4 * (descs[r].n_seq + 1),
                     cudaMemcpyDeviceToHost) != cudaSuccess)
        return RELKL_ERR_CUDA;
      op[r] = offs[r].data();
    }
  }
  (void)part;
  char why[256];
  return relkl_check_schedule(n_rel, descs, bwd ? 1 : 0, n_parts, lp, op, why, sizeof why);
}
#endif

relkl_status fwd_impl(int32_t n_rel, const relkl_desc* descs, const void* const* x_t,
                      const void* const* x_s, float* const* kl, float* const* stats, int32_t part,
                      int32_t n_parts, void* ws, size_t ws_bytes, void* stream) {
  if (n_parts < 1 || part < 0 || part >= n_parts) return RELKL_ERR_INVALID;
  bool empty = false;
  relkl_status s = check_multi(n_rel, descs, x_t, x_s, &empty);
  if (s != RELKL_OK || empty) return s;
  if (!kl || !stats) return RELKL_ERR_INVALID;
  for (int r = 0; r < n_rel; ++r)
    if (n_units(descs[r]) && (!kl[r] || !stats[r] || !aligned(kl[r], 4) || !aligned(stats[r], 16)))
      return RELKL_ERR_INVALID;
  if ((s = check_ws(ws, ws_bytes)) != RELKL_OK) return s;
  DevInfo dev;
  if ((s = device_info(&dev)) != RELKL_OK) return s;
  if (dev.major != 10) return RELKL_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (use_tc(n_rel, descs, x_t, x_s)) {
#ifdef RELKL_CHECKS
    if ((s = debug_schedule_check(n_rel, descs, false, part, n_parts)) != RELKL_OK) return s;
#endif
    TcParams p;
    if ((s = build_tc(n_rel, descs, x_t, x_s, &p, ws, part, n_parts)) != RELKL_OK) return s;
    set_seg_outputs(&p, n_rel, descs, kl, stats, nullptr, nullptr, nullptr);
    if (p.n_items == 0) return RELKL_OK;   // this part holds no work item
    const int grid = p.n_items < dev.sms ? p.n_items : dev.sms;
    e = tc_launch_fwd(p, descs[0].d, grid, st);
  } else {
    SimtParams p;
    build_simt(n_rel, descs, x_t, x_s, &p, part, n_parts);
    set_seg_outputs(&p, n_rel, descs, kl, stats, nullptr, nullptr, nullptr);
    e = simt_launch_fwd(p, st);
  }
  return e == cudaSuccess ? RELKL_OK : cuda_fail(e);
}

relkl_status bwd_impl(int32_t n_rel, const relkl_desc* descs, const void* const* x_t,
                      const void* const* x_s, const float* const* stats, const float* const* dkl,
                      float* const* dx_s, int32_t part, int32_t n_parts, void* ws,
                      size_t ws_bytes, void* stream) {
  if (n_parts < 1 || part < 0 || part >= n_parts) return RELKL_ERR_INVALID;
  bool empty = false;
  relkl_status s = check_multi(n_rel, descs, x_t, x_s, &empty);
  if (s != RELKL_OK || empty) return s;
  if (!stats || !dx_s) return RELKL_ERR_INVALID;
  for (int r = 0; r < n_rel; ++r) {
    if (!n_units(descs[r])) continue;
    if (!stats[r] || !dx_s[r] || !aligned(stats[r], 16) || !aligned(dx_s[r], 16))
      return RELKL_ERR_INVALID;
    if (dkl && dkl[r] && !aligned(dkl[r], 4)) return RELKL_ERR_INVALID;
  }
  if ((s = check_ws(ws, ws_bytes)) != RELKL_OK) return s;
  DevInfo dev;
  if ((s = device_info(&dev)) != RELKL_OK) return s;
  if (dev.major != 10) return RELKL_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  const bool tc = use_tc(n_rel, descs, x_t, x_s);
  TcParams tp;
  SimtParams sp;
  if (tc) {
#ifdef RELKL_CHECKS
    if ((s = debug_schedule_check(n_rel, descs, true, part, n_parts)) != RELKL_OK) return s;
#endif
    if ((s = build_tc(n_rel, descs, x_t, x_s, &tp, ws, part, n_parts)) != RELKL_OK) return s;
    set_seg_outputs(&tp, n_rel, descs, nullptr, nullptr, stats, dkl, dx_s);
    for (int r = 0, seg = 0; r < n_rel; ++r) {
      if (!n_units(descs[r])) continue;
      TcSeg& sg = tp.seg[seg++];
      if ((s = encode_dx(&sg.tm_dx, descs[r], dx_s[r])) != RELKL_OK) return s;
      // 64-row boxes for the column tiles of the d = 128 backward
      if ((s = encode_x(&sg.tm_t64, descs[r], x_t[r], 64)) != RELKL_OK) return s;
      if ((s = encode_x(&sg.tm_s64, descs[r], x_s[r], 64)) != RELKL_OK) return s;
    }
  } else {
    build_simt(n_rel, descs, x_t, x_s, &sp, part, n_parts);
    set_seg_outputs(&sp, n_rel, descs, nullptr, nullptr, stats, dkl, dx_s);
  }
  // dX_s is accumulated by reduce-adds in L2: clear it first (same stream)
  for (int r = 0; r < n_rel; ++r) {
    if (!n_units(descs[r])) continue;
    // the whole [B, H, N, d] tensor (packed sequences: B = 1, every token)
    const int64_t n = static_cast<int64_t>(descs[r].B) * descs[r].H * descs[r].N * descs[r].d;
    if ((e = launch_zero(dx_s[r], n, dev.sms, st)) != cudaSuccess) return cuda_fail(e);
  }
  if (tc) {
    // the launcher sizes the grid (at most one CTA per SM) from the work items
    // of the kernel it picks; a part without items launches nothing
    e = tc_launch_bwd(tp, descs[0].d, dev.sms, st);
  } else {
    e = simt_launch_bwd(sp, st);
  }
  return e == cudaSuccess ? RELKL_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

relkl_status relkl_fwd_qkv(int32_t n_rel, const relkl_desc* descs, const void* const* x_t,
                           const void* const* x_s, float* const* kl, float* const* stats,
                           void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("relkl_fwd_qkv");
  return fwd_impl(n_rel, descs, x_t, x_s, kl, stats, 0, 1, ws, ws_bytes, stream);
}

relkl_status relkl_bwd_qkv(int32_t n_rel, const relkl_desc* descs, const void* const* x_t,
                           const void* const* x_s, const float* const* stats,
                           const float* const* dkl, float* const* dx_s, void* ws,
                           size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("relkl_bwd_qkv");
  return bwd_impl(n_rel, descs, x_t, x_s, stats, dkl, dx_s, 0, 1, ws, ws_bytes, stream);
}

relkl_status relkl_fwd_qkv_part(int32_t n_rel, const relkl_desc* descs, const void* const* x_t,
                                const void* const* x_s, float* const* kl, float* const* stats,
                                int32_t part, int32_t n_parts, void* ws, size_t ws_bytes,
                                void* stream) {
  NvtxRange nvtx_range("relkl_fwd_qkv_part");
  return fwd_impl(n_rel, descs, x_t, x_s, kl, stats, part, n_parts, ws, ws_bytes, stream);
}

relkl_status relkl_bwd_qkv_part(int32_t n_rel, const relkl_desc* descs, const void* const* x_t,
                                const void* const* x_s, const float* const* stats,
                                const float* const* dkl, float* const* dx_s, int32_t part,
                                int32_t n_parts, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("relkl_bwd_qkv_part");
  return bwd_impl(n_rel, descs, x_t, x_s, stats, dkl, dx_s, part, n_parts, ws, ws_bytes, stream);
}

relkl_status relkl_fwd(const relkl_desc* desc, const void* x_t, const void* x_s, float* kl,
                       float* stats, void* ws, size_t ws_bytes, void* stream) {
  const void* xt[1] = {x_t};
  const void* xs[1] = {x_s};
  float* k[1] = {kl};
  float* st[1] = {stats};
  return relkl_fwd_qkv(1, desc, xt, xs, k, st, ws, ws_bytes, stream);
}

relkl_status relkl_bwd(const relkl_desc* desc, const void* x_t, const void* x_s,
                       const float* stats, const float* dkl, float* dx_s, void* ws,
                       size_t ws_bytes, void* stream) {
  const void* xt[1] = {x_t};
  const void* xs[1] = {x_s};
  const float* st[1] = {stats};
  const float* g[1] = {dkl};
  float* dx[1] = {dx_s};
  return relkl_bwd_qkv(1, desc, xt, xs, st, g, dx, ws, ws_bytes, stream);
}

relkl_status relkl_get_device_error(const void* ws, void* stream, uint32_t* where) {
  if (where) *where = 0;
  relkl_status s = check_ws(ws, kWorkspaceBytes);
  if (s != RELKL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  DevStatus rec;
  e = cudaMemcpy(&rec, ws, sizeof(rec), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (where) *where = rec.where;
  return rec.code == 0 ? RELKL_OK : RELKL_ERR_TIMEOUT;
}

uint64_t relkl_set_wait_timeout_ns(uint64_t ns) { return g_timeout_ns.exchange(ns); }

const char* relkl_status_string(relkl_status s) {
  switch (s) {
    case RELKL_OK: return "RELKL_OK";
    case RELKL_ERR_INVALID: return "RELKL_ERR_INVALID: invalid argument";
    case RELKL_ERR_UNSUPPORTED: return "RELKL_ERR_UNSUPPORTED: unsupported shape, layout or device";
    case RELKL_ERR_CUDA: return "RELKL_ERR_CUDA: a CUDA call failed";
    case RELKL_ERR_WORKSPACE: return "RELKL_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case RELKL_ERR_TIMEOUT: return "RELKL_ERR_TIMEOUT: a bounded device wait ran out";
  }
  return "RELKL_ERR_UNKNOWN";
}

int32_t relkl_last_cuda_error(void) { return g_last_cuda; }

relkl_status relkl_check_schedule(int32_t n_rel, const relkl_desc* descs, int32_t is_bwd,
                                  int32_t n_parts, const int32_t* const* host_lengths,
                                  const int32_t* const* host_cu_seqlens, char* why,
                                  size_t why_len) {
  if (why && why_len) why[0] = 0;
  if (n_rel < 1 || n_rel > kMaxSeg || !descs || n_parts < 1) return RELKL_ERR_INVALID;
  int64_t units = 0;
  for (int r = 0; r < n_rel; ++r) {
    relkl_status s = check_desc(&descs[r]);
    if (s != RELKL_OK) return s;
    if (descs[r].N != descs[0].N || descs[r].causal != descs[0].causal ||
        (descs[r].cu_seqlens == nullptr) != (descs[0].cu_seqlens == nullptr) ||
        descs[r].max_seqlen != descs[0].max_seqlen || descs[r].d != descs[0].d)
      return RELKL_ERR_INVALID;
    if ((descs[r].lengths && (!host_lengths || !host_lengths[r])) ||
        (descs[r].cu_seqlens && (!host_cu_seqlens || !host_cu_seqlens[r])))
      return RELKL_ERR_INVALID;
    units += n_units(descs[r]);
  }
  if (!tc_shape(descs[0])) return RELKL_ERR_UNSUPPORTED;
  if (units == 0 || descs[0].N == 0) return RELKL_OK;
  TcParams p;
  fill_schedule(n_rel, descs, &p, 0, 1);
  // host copies in the launch's segment order (relations without units have none)
  const int* lens[kMaxSeg] = {nullptr, nullptr, nullptr};
  const int* offs[kMaxSeg] = {nullptr, nullptr, nullptr};
  for (int r = 0, seg = 0; r < n_rel; ++r) {
    if (n_units(descs[r]) == 0) continue;
    lens[seg] = host_lengths ? host_lengths[r] : nullptr;
    offs[seg] = host_cu_seqlens ? host_cu_seqlens[r] : nullptr;
    ++seg;
  }
  return schedule_check(p, descs[0].d, is_bwd != 0, n_parts, lens, offs, why, why_len) == 0
             ? RELKL_OK
             : RELKL_ERR_INVALID;
}

int32_t relkl_bwd_kernel_for(int32_t n_rel, const relkl_desc* descs, int32_t n_sms) {
  if (n_rel < 1 || n_rel > kMaxSeg || !descs || n_sms < 1) return 0;
  for (int r = 0; r < n_rel; ++r) {
    if (check_desc(&descs[r]) != RELKL_OK) return 0;
    if (descs[r].N != descs[0].N || descs[r].causal != descs[0].causal ||
        (descs[r].cu_seqlens == nullptr) != (descs[0].cu_seqlens == nullptr) ||
        descs[r].max_seqlen != descs[0].max_seqlen || descs[r].d != descs[0].d)
      return 0;
  }
  if (!tc_shape(descs[0])) return 1;
  TcParams p;
  fill_schedule(n_rel, descs, &p, 0, 1);
  return tc_bwd_kind(p, descs[0].d, n_sms);
}

relkl_status relkl_rope_bwd(int32_t B, int32_t H, int32_t N, int32_t d, const float* dx_post,
                            const relkl_rope* rope, int32_t out_dtype, void* dx_pre,
                            void* stream) {
  NvtxRange nvtx_range("relkl_rope_bwd");
  if (!rope || B < 0 || H < 0 || N < 0 || d < 2 || d > 512 || (d & 1)) return RELKL_ERR_INVALID;
  if (out_dtype != RELKL_BF16 && out_dtype != RELKL_FP32) return RELKL_ERR_INVALID;
  if (rope->reserved != 0 || (rope->apply != 0 && rope->apply != 1)) return RELKL_ERR_INVALID;
  if (!std::isfinite(rope->base) || !(rope->base > 1.0) || !std::isfinite(rope->pos_scale) ||
      !std::isfinite(rope->pos_offset))
    return RELKL_ERR_INVALID;
  const long long tokens = static_cast<long long>(B) * N;
  if (tokens == 0 || H == 0) return RELKL_OK;
  if (tokens > 0x7fffffffLL) return RELKL_ERR_INVALID;
  if (!dx_post || !dx_pre || !aligned(dx_post, 4) || !aligned(dx_pre, out_dtype == RELKL_BF16 ? 2 : 4))
    return RELKL_ERR_INVALID;
  cudaError_t e = launch_rope_bwd(dx_post, dx_pre, B, H, N, d, out_dtype == RELKL_BF16, rope->base,
                                  rope->pos_scale, rope->pos_offset, rope->apply,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RELKL_OK : cuda_fail(e);
}

relkl_status relkl_cast_bf16(const float* src, void* dst, int64_t n, void* stream) {
  NvtxRange nvtx_range("relkl_cast_bf16");
  if (n < 0) return RELKL_ERR_INVALID;
  if (n == 0) return RELKL_OK;
  if (!src || !dst || !aligned(src, 4) || !aligned(dst, 2)) return RELKL_ERR_INVALID;
  // the two ranges may not overlap
  const char* a = reinterpret_cast<const char*>(src);
  const char* b = static_cast<const char*>(dst);
  if (a < b + 2 * n && b < a + 4 * n) return RELKL_ERR_INVALID;
  relkl_status s;
  DevInfo dev;
  if ((s = device_info(&dev)) != RELKL_OK) return s;
  cudaError_t e = launch_cast_bf16(src, dst, n, dev.sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RELKL_OK : cuda_fail(e);
}

relkl_status relkl_weight_grad(int64_t rows, int32_t D, int32_t cols, const void* h,
                               const void* dx_pre, float* dw, void* ws, size_t ws_bytes,
                               void* stream) {
  NvtxRange nvtx_range("relkl_weight_grad");
  if (rows < 1 || rows > 0x7fffffffLL || D < 1 || cols < 1 || (D % 8) || (cols % 8))
    return RELKL_ERR_INVALID;
  if (!h || !dx_pre || !dw || !aligned(h, 16) || !aligned(dx_pre, 16) || !aligned(dw, 16))
    return RELKL_ERR_INVALID;
  relkl_status s = check_ws(ws, ws_bytes);
  if (s != RELKL_OK) return s;
  DevInfo dev;
  if ((s = device_info(&dev)) != RELKL_OK) return s;
  if (dev.major != 10) return RELKL_ERR_UNSUPPORTED;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return RELKL_ERR_CUDA;
  const int r = launch_wgrad(enc, rows, D, cols, h, dx_pre, dw, dev.sms,
                             reinterpret_cast<DevStatus*>(ws), g_timeout_ns.load(),
                             static_cast<cudaStream_t>(stream));
  if (r == 1) return RELKL_ERR_UNSUPPORTED;
  if (r != 0) return cuda_fail(static_cast<cudaError_t>(r - 2));
  return RELKL_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// relkl_fwd_noalloc: the tensor-core forward with its scratch (the device
// status record) in a static device array instead of a caller workspace.
// Host code must not hand the array's name to a kernel: on the host it is a
// stand-in, not a device address.  The address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[RELKL_NOALLOC_SCRATCH_BYTES];

namespace {
// One slot per device index: the array's device address and the context it
// was looked up in.  A context torn down and created again (cudaDeviceReset,
// or a reset after a sticky error) loads the module again, possibly at another
// address, so a slot is only reused while the device's current context is the
// one recorded in it.
struct NoallocSlot {
  CUcontext ctx;
  void* addr;
};
NoallocSlot g_noalloc[64];
std::mutex g_noalloc_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn g_ctx_current = nullptr;
std::once_flag g_ctx_once;

CUcontext current_context() {
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(fn);
  });
  CUcontext c = nullptr;
  if (g_ctx_current && g_ctx_current(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}

relkl_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return RELKL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc[dev];
  const CUcontext ctx = current_context();
  if (!slot.addr || ctx != slot.ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    slot.addr = p;
    slot.ctx = current_context();   // the lookup made the device's context current
  }
  *out = slot.addr;
  return RELKL_OK;
}
}  // namespace

extern "C" relkl_status relkl_fwd_noalloc(const relkl_desc* desc, const void* x_t,
                                          const void* x_s, float* kl, float* stats,
                                          void* stream) {
  NvtxRange nvtx_range("relkl_fwd_noalloc");
  const void* xt[1] = {x_t};
  const void* xs[1] = {x_s};
  bool empty = false;
  relkl_status s = check_multi(1, desc, xt, xs, &empty);
  if (s != RELKL_OK || empty) return s;
  if (!kl || !stats || !aligned(kl, 4) || !aligned(stats, 16)) return RELKL_ERR_INVALID;
  if (!use_tc(1, desc, xt, xs)) return RELKL_ERR_UNSUPPORTED;
  if (kWorkspaceBytes > sizeof(g_noalloc_scratch)) return RELKL_ERR_WORKSPACE;
  DevInfo dev;
  if ((s = device_info(&dev)) != RELKL_OK) return s;
  if (dev.major != 10) return RELKL_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != RELKL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the record keeps the previous call's contents: clear it on this stream first
  cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(DevStatus), st);
  if (e != cudaSuccess) return cuda_fail(e);
  TcParams p;
  if ((s = build_tc(1, desc, xt, xs, &p, scratch)) != RELKL_OK) return s;
  float* k[1] = {kl};
  float* sts[1] = {stats};
  set_seg_outputs(&p, 1, desc, k, sts, nullptr, nullptr, nullptr);
  const int grid = p.n_items < dev.sms ? p.n_items : dev.sms;
  e = tc_launch_fwd(p, desc->d, grid, st);
  return e == cudaSuccess ? RELKL_OK : cuda_fail(e);
}
