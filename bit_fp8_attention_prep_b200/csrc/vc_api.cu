// vc_api.cu -- host side of the C ABI declared in include/vc_attn.h: argument
// validation, workspace carving, TMA descriptor encoding and kernel launches.
// Nothing here allocates device memory or synchronises the device.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <cmath>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/vc_attn.h"
#include "../../include/vc_attn_testing.h"
#include "vc_kernels.h"

namespace {

// An NVTX range over the host side of an ABI call (a profiler's timeline shows
// which call enqueued which kernels). NVTX is header-only: without a tool
// attached a range costs a few nanoseconds.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};  // kernels enqueued by this library since load

vc_status_t fail(vc_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

vc_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(VC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int nblocks(int S) { return (S + 127) / 128; }

vc_status_t check_shape(const vc_shape_t* sh) {
  if (!sh) return fail(VC_ERR_INVALID_ARG, "shape is NULL");
  if (sh->D != 128) return fail(VC_ERR_INVALID_ARG, "D must be 128 (got %d)", sh->D);
  if (sh->B < 1 || sh->S < 1 || sh->H < 1)
    return fail(VC_ERR_INVALID_ARG, "B, S, H must be >= 1 (got %d, %d, %d)", sh->B, sh->S, sh->H);
  if (sh->dtype != VC_DTYPE_F16 && sh->dtype != VC_DTYPE_BF16)
    return fail(VC_ERR_INVALID_ARG, "dtype must be VC_DTYPE_F16 or VC_DTYPE_BF16 (got %d)", sh->dtype);
  const long long n = (long long)sh->B * sh->H * nblocks(sh->S) * 128 * 128;
  if (n >= (1ll << 31)) return fail(VC_ERR_INVALID_ARG, "B*H*S_pad*128 = %lld exceeds 2^31", n);
  // every kernel takes one grid row (blockIdx.y) per (b, h) slice
  if ((long long)sh->B * sh->H > 65535)
    return fail(VC_ERR_UNSUPPORTED, "B*H = %lld exceeds 65535 slices", (long long)sh->B * sh->H);
  return VC_OK;
}

vc_status_t check_cfg(const vc_vsmooth_cfg_t* cfg) {
  if (!cfg) return fail(VC_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->mode != VC_MODE_VSMOOTH && cfg->mode != VC_MODE_MEANONLY && cfg->mode != VC_MODE_NAIVE)
    return fail(VC_ERR_INVALID_ARG, "mode must be VC_MODE_VSMOOTH, VC_MODE_MEANONLY or VC_MODE_NAIVE (got %d)",
                cfg->mode);
  if (cfg->mode == VC_MODE_VSMOOTH) {
    if (cfg->k < 1 || cfg->k > vc::kMaxClusters)
      return fail(VC_ERR_INVALID_ARG, "k must be in [1, %d] (got %d)", vc::kMaxClusters, cfg->k);
    if (cfg->iters < 1 || cfg->iters > 64) return fail(VC_ERR_INVALID_ARG, "iters must be in [1, 64] (got %d)", cfg->iters);
  }
  if (cfg->residual_fmt != VC_RESIDUAL_E4M3 && cfg->residual_fmt != VC_RESIDUAL_NVFP4 &&
      cfg->residual_fmt != VC_RESIDUAL_E4M3_PER_CHANNEL && cfg->residual_fmt != VC_RESIDUAL_MXFP4)
    return fail(VC_ERR_INVALID_ARG,
                "residual_fmt must be VC_RESIDUAL_E4M3, _NVFP4, _E4M3_PER_CHANNEL or _MXFP4 (got %d)",
                cfg->residual_fmt);
  return VC_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout of vc_attn_prepare_v (every piece 256-B aligned).
struct WsLayout {
  size_t cent, sums, counts, assign, assign2, hist, offs, amax, cops, work, total;
};

WsLayout ws_layout(const vc_shape_t* sh, const vc_vsmooth_cfg_t* cfg) {
  const size_t BH = (size_t)sh->B * sh->H;
  const size_t k = cfg->mode == VC_MODE_VSMOOTH ? (size_t)cfg->k : 1;
  const size_t nch = (size_t)((sh->S + vc::kChunk - 1) / vc::kChunk);
  WsLayout w;
  size_t off = 0;
  w.cent = off;   off += align256(BH * k * 128 * 4);
  w.sums = off;   off += align256(BH * k * 128 * 8);
  w.counts = off; off += align256(BH * k * 4);
  w.assign = off; off += align256(BH * (size_t)sh->S);
  w.assign2 = off; off += cfg->mode == VC_MODE_VSMOOTH ? align256(BH * (size_t)sh->S) : 0;
  w.hist = off;   off += align256(BH * nch * k * 4);
  w.offs = off;   off += align256(BH * nch * k * 4);
  // residual amax: one per (b, h), or one per (b, h, channel)
  w.amax = off;   off += align256(BH * 4 * (cfg->residual_fmt == VC_RESIDUAL_E4M3_PER_CHANNEL ? 128 : 1));
  // the tensor-core k-means assignment (BF16 V): centroid operand blocks and the
  // passes' work counters
  const bool tc = cfg->mode == VC_MODE_VSMOOTH && sh->dtype == VC_DTYPE_BF16;
  w.cops = off;   off += tc ? align256(BH * vc::tc_cops_bytes((int)k)) : 0;
  w.work = off;   off += tc ? align256(sizeof(int) * (size_t)cfg->iters) : 0;
  w.total = off;
  return w;
}

// Per-device one-time set-up: the device must be sm_100 and the kernels' shared
// memory limits raised.
std::mutex g_mu;
int g_ready[64];  // 0 unknown, 1 ready, -1 unsupported

vc_status_t ensure_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(VC_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_ready[dev] == 1) return VC_OK;
  if (g_ready[dev] == -1) return fail(VC_ERR_UNSUPPORTED, "device %d is not an sm_100 GPU", dev);
  int major = 0, minor = 0;
  if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute");
  if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute");
  if (major != 10 || minor != 0) {
    g_ready[dev] = -1;
    return fail(VC_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev, major, minor);
  }
  if ((e = vc::prep_configure()) != cudaSuccess) return cuda_fail(e, "configuring prep kernels");
  if ((e = vc::attn_configure()) != cudaSuccess) return cuda_fail(e, "configuring attention kernel");
  g_ready[dev] = 1;
  return VC_OK;
}

// Number of SMs of the current device (cached per device; 148 if the query fails).
int g_sms[64];
int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (g_sms[dev] == 0) {
    int n = 0;
    g_sms[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
  }
  return g_sms[dev];
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D uint8 tensor map: rows of `inner` bytes, `rows` rows, 128 x 128 byte box,
// 128-byte swizzle (the canonical K-major UMMA operand layout).
vc_status_t make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(VC_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(VC_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return VC_OK;
}

}  // namespace

extern "C" {

int32_t vc_attn_version(void) { return 100; }

const char* vc_attn_last_error(void) { return g_last_error.c_str(); }

uint64_t vc_attn_launch_count(void) { return g_launches.load(); }

size_t vc_attn_prepare_v_workspace_bytes(const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg) {
  if (check_shape(shape) != VC_OK || check_cfg(cfg) != VC_OK) return 0;
  return ws_layout(shape, cfg).total;
}

}  // extern "C"

// Shape, config and output-pointer checks shared by the prep entry points.
static vc_status_t check_prep_args(const void* v, const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                                   const vc_prepared_v_t* out) {
  vc_status_t st;
  if ((st = check_shape(shape)) != VC_OK) return st;
  if ((st = check_cfg(cfg)) != VC_OK) return st;
  if (!v || !out || !out->perm || !out->mu || !out->v_codes || !out->s_v)
    return fail(VC_ERR_INVALID_ARG, "v, out, out->perm, out->mu, out->v_codes and out->s_v must be non-NULL");
  if ((cfg->residual_fmt == VC_RESIDUAL_NVFP4 || cfg->residual_fmt == VC_RESIDUAL_MXFP4) && !out->v_scales)
    return fail(VC_ERR_INVALID_ARG, "out->v_scales must be non-NULL for the NVFP4 and MXFP4 residuals");
  if (!aligned16(v) || !aligned16(out->perm) || !aligned16(out->mu) || !aligned16(out->v_codes) ||
      !aligned16(out->s_v) || (out->v_scales && !aligned16(out->v_scales)))
    return fail(VC_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  return VC_OK;
}

// vc_attn_prepare_v where slice (b, h) of this call is slice (seed_b0 + b,
// seed_h0 + h) of a problem with seed_H heads (whose k-means seed it takes).
static vc_status_t prepare_v_impl(const void* v, const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                                  const vc_prepared_v_t* out, void* workspace, size_t workspace_bytes,
                                  uint8_t* assign_history, void* stream, int seed_H, int seed_b0, int seed_h0) {
  vc_status_t st;
  if ((st = check_prep_args(v, shape, cfg, out)) != VC_OK) return st;
  const WsLayout w = ws_layout(shape, cfg);
  if (!workspace || workspace_bytes < w.total)
    return fail(VC_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.total,
                workspace ? workspace_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VC_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((st = ensure_device()) != VC_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  vc::PrepPlan pl;
  pl.B = shape->B;
  pl.S = shape->S;
  pl.H = shape->H;
  pl.k = cfg->mode == VC_MODE_VSMOOTH ? cfg->k : 1;
  pl.iters = cfg->iters;
  pl.fmt = cfg->residual_fmt;
  pl.mode = cfg->mode;
  pl.seed = cfg->seed;
  pl.seed_H = seed_H;
  pl.seed_b0 = seed_b0;
  pl.seed_h0 = seed_h0;
  pl.nb = nblocks(shape->S);
  pl.S_pad = pl.nb * 128;
  pl.nchunks = (shape->S + vc::kChunk - 1) / vc::kChunk;
  pl.cent = reinterpret_cast<float*>(ws + w.cent);
  pl.sums = reinterpret_cast<unsigned long long*>(ws + w.sums);
  pl.counts = reinterpret_cast<int*>(ws + w.counts);
  pl.assign = ws + w.assign;
  pl.assign2 = ws + w.assign2;
  pl.hist = reinterpret_cast<int*>(ws + w.hist);
  pl.offs = reinterpret_cast<int*>(ws + w.offs);
  pl.amax = reinterpret_cast<unsigned int*>(ws + w.amax);
  // BF16 V: the k-means distances run on the tensor cores, which read V through
  // a 3D tensor map [B*S][H][128] (boxes of 128 tokens x 1 head x 64 dims)
  pl.tc_assign = shape->dtype == VC_DTYPE_BF16 && cfg->mode == VC_MODE_VSMOOTH;
  pl.num_sms = device_sms();
  pl.cops = ws + w.cops;
  pl.work = reinterpret_cast<int*>(ws + w.work);
  if (pl.tc_assign) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(VC_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[3] = {128, (cuuint64_t)shape->H, (cuuint64_t)shape->B * (cuuint64_t)shape->S};
    const cuuint64_t strides[2] = {256, (cuuint64_t)shape->H * 256};
    const cuuint32_t box[3] = {64, 1, 128};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(&pl.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(v), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(VC_ERR_CUDA, "cuTensorMapEncodeTiled (V for the k-means) failed (%d)", (int)r);
  }
  int nl = 0;
  cudaError_t e =
      vc::launch_prepare_v(v, shape->dtype, pl, *out, assign_history, static_cast<cudaStream_t>(stream), &nl);
  g_launches += (uint64_t)nl;
  if (e != cudaSuccess) return cuda_fail(e, "launching V-Smooth prep");
  return VC_OK;
}

extern "C" {

size_t vc_attn_prepare_v_repair_workspace_bytes(const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg) {
  if (check_shape(shape) != VC_OK || check_cfg(cfg) != VC_OK) return 0;
  const size_t BH = (size_t)shape->B * shape->H;
  return ws_layout(shape, cfg).total + align256(BH * (size_t)shape->S * 4) + align256(BH * 8);
}

vc_status_t vc_attn_prepare_v_repair(const void* v, const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                                     double budget, const vc_prepared_v_t* out, uint8_t* kept, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  NvtxRange range("vc_attn_prepare_v_repair");
  g_last_error.clear();
  vc_status_t st;
  if ((st = check_shape(shape)) != VC_OK) return st;
  if ((st = check_cfg(cfg)) != VC_OK) return st;
  if (cfg->residual_fmt != VC_RESIDUAL_E4M3)
    return fail(VC_ERR_UNSUPPORTED, "the residual repair is defined for the E4M3 residual only");
  if (!(budget >= 0.0 && budget <= 1.0)) return fail(VC_ERR_INVALID_ARG, "budget must be in [0, 1]");
  const size_t need = vc_attn_prepare_v_repair_workspace_bytes(shape, cfg);
  if (!workspace || workspace_bytes < need)
    return fail(VC_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                workspace ? workspace_bytes : (size_t)0);
  const WsLayout w = ws_layout(shape, cfg);
  if ((st = prepare_v_impl(v, shape, cfg, out, workspace, w.total, nullptr, stream, shape->H, 0, 0)) != VC_OK)
    return st;
  const size_t BH = (size_t)shape->B * shape->H;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* err = reinterpret_cast<float*>(ws + w.total);
  unsigned long long* thr = reinterpret_cast<unsigned long long*>(ws + w.total + align256(BH * (size_t)shape->S * 4));
  const int m = (int)std::min<double>((double)shape->S, std::ceil(budget * (double)shape->S));
  int n = 0;
  cudaError_t e = vc::launch_repair(v, shape->dtype, shape->B, shape->S, shape->H, out->perm, out->mu,
                                    reinterpret_cast<const unsigned int*>(ws + w.amax), out->v_codes, m, err, thr, kept,
                                    static_cast<cudaStream_t>(stream), &n);
  g_launches += (uint64_t)n;
  if (e != cudaSuccess) return cuda_fail(e, "launching the residual repair");
  return VC_OK;
}

vc_status_t vc_attn_prepare_v(const void* v, const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                              const vc_prepared_v_t* out, void* workspace, size_t workspace_bytes,
                              uint8_t* assign_history, void* stream) {
  NvtxRange range("vc_attn_prepare_v");
  g_last_error.clear();
  return prepare_v_impl(v, shape, cfg, out, workspace, workspace_bytes, assign_history, stream, shape ? shape->H : 0,
                        0, 0);
}

vc_status_t vc_attn_prepare_v_shard(const void* v, const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                                    int32_t h_base, int32_t H_total, const vc_prepared_v_t* out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  NvtxRange range("vc_attn_prepare_v_shard");
  g_last_error.clear();
  vc_status_t st;
  if ((st = check_shape(shape)) != VC_OK) return st;
  if (h_base < 0 || H_total < 1 || (long long)h_base + shape->H > (long long)H_total)
    return fail(VC_ERR_INVALID_ARG, "heads [h_base, h_base + H) = [%d, %lld) must lie in [0, H_total = %d)", h_base,
                (long long)h_base + shape->H, H_total);
  if ((long long)shape->B * H_total > 0x7fffffffll)
    return fail(VC_ERR_INVALID_ARG, "B * H_total exceeds the slice index range");
  return prepare_v_impl(v, shape, cfg, out, workspace, workspace_bytes, nullptr, stream, H_total, 0, h_base);
}

vc_status_t vc_attn_quant_qk(const void* q, const void* k, const vc_shape_t* shape, const int32_t* perm,
                             const vc_qk_fp8_t* out, void* stream) {
  NvtxRange range("vc_attn_quant_qk");
  g_last_error.clear();
  vc_status_t st;
  if ((st = check_shape(shape)) != VC_OK) return st;
  if (!q || !k || !perm || !out || !out->q_codes || !out->q_scales || !out->k_codes || !out->k_scales)
    return fail(VC_ERR_INVALID_ARG, "q, k, perm, out and every field of out must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(perm) || !aligned16(out->q_codes) || !aligned16(out->k_codes) ||
      !aligned16(out->q_scales) || !aligned16(out->k_scales))
    return fail(VC_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if ((st = ensure_device()) != VC_OK) return st;
  int n = 0;
  cudaError_t e = vc::launch_quant_qk(q, k, shape->dtype, shape->B, shape->S, shape->H, perm, *out, nullptr,
                                      nullptr, static_cast<cudaStream_t>(stream), &n);
  g_launches += n;
  if (e != cudaSuccess) return cuda_fail(e, "launching Q/K quantisation");
  return VC_OK;
}

size_t vc_attn_quant_qk_smoothk_workspace_bytes(const vc_shape_t* shape) {
  if (check_shape(shape) != VC_OK) return 0;
  // the int64 token sums, then the fp32 means
  return (sizeof(unsigned long long) + sizeof(float)) * (size_t)shape->B * shape->H * 128;
}

vc_status_t vc_attn_quant_qk_smoothk(const void* q, const void* k, const vc_shape_t* shape, const int32_t* perm,
                                     const vc_qk_fp8_t* out, void* workspace, size_t workspace_bytes,
                                     float* k_mean, void* stream) {
  NvtxRange range("vc_attn_quant_qk_smoothk");
  g_last_error.clear();
  vc_status_t st;
  if ((st = check_shape(shape)) != VC_OK) return st;
  if (!q || !k || !perm || !out || !out->q_codes || !out->q_scales || !out->k_codes || !out->k_scales)
    return fail(VC_ERR_INVALID_ARG, "q, k, perm, out and every field of out must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(perm) || !aligned16(out->q_codes) || !aligned16(out->k_codes) ||
      !aligned16(out->q_scales) || !aligned16(out->k_scales) || !aligned16(k_mean))
    return fail(VC_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  const size_t need = vc_attn_quant_qk_smoothk_workspace_bytes(shape);
  if (!workspace || workspace_bytes < need)
    return fail(VC_ERR_WORKSPACE, "K smoothing needs %zu bytes of workspace (got %zu)", need,
                workspace ? workspace_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(VC_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if ((st = ensure_device()) != VC_OK) return st;
  int n = 0;
  cudaError_t e = vc::launch_quant_qk(q, k, shape->dtype, shape->B, shape->S, shape->H, perm, *out,
                                      static_cast<unsigned long long*>(workspace), k_mean,
                                      static_cast<cudaStream_t>(stream), &n);
  g_launches += n;
  if (e != cudaSuccess) return cuda_fail(e, "launching the smoothed Q/K quantisation");
  return VC_OK;
}

vc_status_t vc_attn_residual_energy(const void* v, const vc_shape_t* shape, const int32_t* perm, const float* mu,
                                    double* energy, void* stream) {
  NvtxRange range("vc_attn_residual_energy");
  g_last_error.clear();
  vc_status_t st;
  if ((st = check_shape(shape)) != VC_OK) return st;
  if (!v || !energy) return fail(VC_ERR_INVALID_ARG, "v and energy must be non-NULL");
  if (!aligned16(v) || !aligned16(perm) || !aligned16(mu) || !aligned16(energy))
    return fail(VC_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if ((st = ensure_device()) != VC_OK) return st;
  cudaError_t e = vc::launch_residual_energy(v, shape->dtype, shape->B, shape->S, shape->H, perm, mu, energy,
                                             static_cast<cudaStream_t>(stream));
  g_launches += 1;
  if (e != cudaSuccess) return cuda_fail(e, "launching the residual-energy reduction");
  return VC_OK;
}

// 2D tensor map over packed E2M1 codes (two per byte): rows of `inner` codes,
// `rows` rows, 128 x 128 code box, each 16 codes widened by the TMA into a
// 16-byte shared-memory container (the 8-bit operand footprint of
// kind::mxf8f6f4), 128-byte swizzle. The base must be 32-byte aligned and
// inner a multiple of 128.
static vc_status_t make_map_e2m1(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(VC_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner / 2};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(VC_ERR_CUDA, "cuTensorMapEncodeTiled (E2M1) failed (%d)", (int)r);
  return VC_OK;
}

// Which attention kernel a forward call runs.
enum class FwdKind {
  E4M3,         // one E4M3 plane, s_V per (b, h)
  E4M3_EXP2,    // the same with ex2 + E4M3 conversion in place of ExpCast (test hook)
  E4M3_CHANNEL, // one E4M3 plane, s_V per (b, h, channel)
  NVFP4,        // pv's NVFP4 residual split into two E4M3 planes in `workspace`, value scale 8 g
  TWO_PLANES,   // pv->v_codes already holds two E4M3 planes at s_V (the repaired residual)
  MXFP4         // E2M1 codes with power-of-two scales, block-scaled PV
};

static vc_status_t forward_common(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv, const vc_shape_t* shape,
                                  float softmax_scale, int32_t k_p, void* o, int32_t* dev_status, void* stream,
                                  FwdKind kind, void* workspace = nullptr, size_t workspace_bytes = 0) {
  const bool nvfp4 = kind == FwdKind::NVFP4;
  g_last_error.clear();
  vc_status_t st;
  if ((st = check_shape(shape)) != VC_OK) return st;
  if (!qk || !pv || !o) return fail(VC_ERR_INVALID_ARG, "qk, pv and o must be non-NULL");
  if (!qk->q_codes || !qk->q_scales || !qk->k_codes || !qk->k_scales || !pv->mu || !pv->v_codes || !pv->s_v)
    return fail(VC_ERR_INVALID_ARG, "a required field of qk or pv is NULL");
  if ((nvfp4 || kind == FwdKind::MXFP4) && (!pv->v_scales || !aligned16(pv->v_scales)))
    return fail(VC_ERR_INVALID_ARG, "pv->v_scales must be non-NULL and 16-byte aligned for NVFP4 and MXFP4");
  if (kind == FwdKind::MXFP4 && (reinterpret_cast<uintptr_t>(pv->v_codes) & 31u) != 0)
    return fail(VC_ERR_INVALID_ARG, "pv->v_codes must be 32-byte aligned for the MXFP4 residual");
  if (!aligned16(o) || !aligned16(qk->q_codes) || !aligned16(qk->k_codes) || !aligned16(pv->v_codes) ||
      !aligned16(pv->mu) || (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)))
    return fail(VC_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.0f) || !(softmax_scale < 1e30f))
    return fail(VC_ERR_INVALID_ARG, "softmax_scale must be positive and finite");
  if (k_p < 0 || k_p > 8) return fail(VC_ERR_INVALID_ARG, "k_p must be in [0, 8] (got %d)", k_p);
  const int nb = nblocks(shape->S), S_pad = nb * 128, BH = shape->B * shape->H;
  if (nvfp4) {
    const size_t need = (size_t)2 * BH * 128 * S_pad;
    if (!workspace || workspace_bytes < need)
      return fail(VC_ERR_WORKSPACE, "NVFP4-V attention needs %zu bytes of workspace (got %zu)", need,
                  workspace ? workspace_bytes : (size_t)0);
    if (!aligned16(workspace)) return fail(VC_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  }
  if ((st = ensure_device()) != VC_OK) return st;
  CUtensorMap tq, tk, tv;
  if ((st = make_map_u8(&tq, qk->q_codes, 128, (uint64_t)BH * S_pad)) != VC_OK) return st;
  if ((st = make_map_u8(&tk, qk->k_codes, 128, (uint64_t)BH * S_pad)) != VC_OK) return st;
  vc::AttnParams p;
  p.B = shape->B;
  p.S = shape->S;
  p.H = shape->H;
  p.nb = nb;
  p.S_pad = S_pad;
  p.q_scales = qk->q_scales;
  p.k_scales = qk->k_scales;
  p.mu = pv->mu;
  p.s_v = pv->s_v;
  p.v_scales = pv->v_scales;
  p.kappa = (float)((double)softmax_scale * 1.4426950408889634);
  p.v_mul = nvfp4 ? 8.0f : 1.0f;
  p.bias_b = 56 + 8 * k_p;
  p.o = o;
  p.status = dev_status;
  p.wait_ns = 2000000000ull;
  cudaError_t e;
  const cudaStream_t cst = static_cast<cudaStream_t>(stream);
  if (kind == FwdKind::TWO_PLANES) {
    if ((st = make_map_u8(&tv, pv->v_codes, (uint64_t)S_pad, (uint64_t)2 * BH * 128)) != VC_OK) return st;
    e = vc::launch_attn_planes(tq, tk, tv, p, cst);
  } else if (kind == FwdKind::E4M3 || kind == FwdKind::E4M3_EXP2) {
    if ((st = make_map_u8(&tv, pv->v_codes, (uint64_t)S_pad, (uint64_t)BH * 128)) != VC_OK) return st;
    e = vc::launch_attn_e4m3(tq, tk, tv, p, cst, kind == FwdKind::E4M3_EXP2);
  } else if (kind == FwdKind::E4M3_CHANNEL) {
    if ((st = make_map_u8(&tv, pv->v_codes, (uint64_t)S_pad, (uint64_t)BH * 128)) != VC_OK) return st;
    e = vc::launch_attn_channel(tq, tk, tv, p, cst);
  } else if (kind == FwdKind::MXFP4) {
    if ((st = make_map_e2m1(&tv, pv->v_codes, (uint64_t)S_pad, (uint64_t)BH * 128)) != VC_OK) return st;
    e = vc::launch_attn_mx(tq, tk, tv, p, cst);
  } else {
    uint8_t* planes = static_cast<uint8_t*>(workspace);
    e = vc::launch_nvfp4_planes(static_cast<const uint8_t*>(pv->v_codes), static_cast<const uint8_t*>(pv->v_scales),
                                BH, S_pad, planes, static_cast<cudaStream_t>(stream));
    g_launches += 1;
    if (e != cudaSuccess) return cuda_fail(e, "launching the NVFP4 plane split");
    if ((st = make_map_u8(&tv, planes, (uint64_t)S_pad, (uint64_t)2 * BH * 128)) != VC_OK) return st;
    e = vc::launch_attn_planes(tq, tk, tv, p, static_cast<cudaStream_t>(stream));
  }
  g_launches += 1;
  if (e != cudaSuccess) return cuda_fail(e, "launching attention");
  return VC_OK;
}

vc_status_t vc_attn_forward(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv, const vc_shape_t* shape,
                            float softmax_scale, int32_t k_p, void* o, int32_t* dev_status, void* stream) {
  NvtxRange range("vc_attn_forward");
  return forward_common(qk, pv, shape, softmax_scale, k_p, o, dev_status, stream, FwdKind::E4M3);
}

vc_status_t vc_attn_forward_e4m3_per_channel(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv,
                                             const vc_shape_t* shape, float softmax_scale, int32_t k_p, void* o,
                                             int32_t* dev_status, void* stream) {
  NvtxRange range("vc_attn_forward_e4m3_per_channel");
  return forward_common(qk, pv, shape, softmax_scale, k_p, o, dev_status, stream, FwdKind::E4M3_CHANNEL);
}

vc_status_t vc_attn_forward_mxfp4v(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv, const vc_shape_t* shape,
                                   float softmax_scale, int32_t k_p, void* o, int32_t* dev_status, void* stream) {
  NvtxRange range("vc_attn_forward_mxfp4v");
  return forward_common(qk, pv, shape, softmax_scale, k_p, o, dev_status, stream, FwdKind::MXFP4);
}

vc_status_t vc_attn_test_forward_exp2(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv, const vc_shape_t* shape,
                                      float softmax_scale, int32_t k_p, void* o, int32_t* dev_status, void* stream) {
  return forward_common(qk, pv, shape, softmax_scale, k_p, o, dev_status, stream, FwdKind::E4M3_EXP2);
}

vc_status_t vc_attn_forward_repair(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv, const vc_shape_t* shape,
                                   float softmax_scale, int32_t k_p, void* o, int32_t* dev_status, void* stream) {
  NvtxRange range("vc_attn_forward_repair");
  return forward_common(qk, pv, shape, softmax_scale, k_p, o, dev_status, stream, FwdKind::TWO_PLANES);
}

size_t vc_attn_forward_nvfp4v_workspace_bytes(const vc_shape_t* shape) {
  if (check_shape(shape) != VC_OK) return 0;
  return (size_t)2 * shape->B * shape->H * 128 * (size_t)(nblocks(shape->S) * 128);
}

vc_status_t vc_attn_forward_nvfp4v(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv, const vc_shape_t* shape,
                                   float softmax_scale, int32_t k_p, void* o, void* workspace,
                                   size_t workspace_bytes, int32_t* dev_status, void* stream) {
  NvtxRange range("vc_attn_forward_nvfp4v");
  return forward_common(qk, pv, shape, softmax_scale, k_p, o, dev_status, stream, FwdKind::NVFP4, workspace,
                        workspace_bytes);
}

// ------------------------------------------------------------ fixed-scratch prep
// vc_attn_prepare_v_noalloc: the same prep with its scratch in this file-scope
// device array instead of a caller workspace. In host code `g_noalloc_scratch`
// names a host-side stand-in, not device memory, so its device address is
// looked up once per device with cudaGetSymbolAddress (with that device current)
// and only that address is handed to the kernels.
}  // extern "C"

namespace {
static __device__ __align__(256) uint8_t g_noalloc_scratch[VC_ATTN_NOALLOC_SCRATCH_BYTES];
std::mutex g_noalloc_mu;
void* g_noalloc_addr[64];  // device address of g_noalloc_scratch, per device (null until set up)
}  // namespace

extern "C" {

vc_status_t vc_attn_prepare_v_noalloc(const void* v, const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                                      const vc_prepared_v_t* out, uint8_t* assign_history, void* stream) {
  NvtxRange range("vc_attn_prepare_v_noalloc");
  g_last_error.clear();
  vc_status_t st;
  // the same checks, in the same order, as vc_attn_prepare_v, before anything
  // touches the device: arguments, the scratch size, then the device itself
  if ((st = check_prep_args(v, shape, cfg, out)) != VC_OK) return st;
  const size_t need = ws_layout(shape, cfg).total;
  if (need > VC_ATTN_NOALLOC_SCRATCH_BYTES)
    return fail(VC_ERR_WORKSPACE,
                "this problem needs %zu bytes of prep scratch; the fixed scratch of vc_attn_prepare_v_noalloc "
                "holds %zu bytes (use vc_attn_prepare_v with a caller workspace)",
                need, (size_t)VC_ATTN_NOALLOC_SCRATCH_BYTES);
  if ((st = ensure_device()) != VC_OK) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(VC_ERR_UNSUPPORTED, "device index %d out of range", dev);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the fixed prep scratch");
      g_noalloc_addr[dev] = p;
    }
    scratch = g_noalloc_addr[dev];
  }
  return vc_attn_prepare_v(v, shape, cfg, out, scratch, VC_ATTN_NOALLOC_SCRATCH_BYTES, assign_history, stream);
}

}  // extern "C"

// ------------------------------------------------------------ host-buffer pipeline
namespace {

// Device workspace of vc_attn_run_host for chunks of at most hc heads of one
// batch entry (every piece 256-B aligned), in two slots used by alternate
// chunks: the chunk's Q, K, V and O buffers (the copies of one chunk overlap the
// compute of the other), then its prepared-V, Q/K code, prep scratch and NVFP4
// plane buffers (the two slots compute on two streams, so that one chunk's
// last wave of attention CTAs shares the GPU with the next chunk's kernels).
struct RunHostLayout {
  size_t in[2][3], out[2];
  size_t perm[2], mu[2], v_codes[2], v_scales[2], s_v[2], q_codes[2], q_scales[2], k_codes[2], k_scales[2];
  size_t prep_ws[2], prep_ws_bytes, planes[2], planes_bytes, total;
};

RunHostLayout run_host_layout(const vc_shape_t* sh, const vc_vsmooth_cfg_t* cfg, int hc) {
  const size_t S = (size_t)sh->S, nb = (size_t)nblocks(sh->S), S_pad = nb * 128, n = (size_t)hc;
  const size_t chunk_bytes = S * n * 128 * 2;
  const int fmt = cfg->residual_fmt;
  const bool nv = fmt == VC_RESIDUAL_NVFP4, mx = fmt == VC_RESIDUAL_MXFP4, ch = fmt == VC_RESIDUAL_E4M3_PER_CHANNEL;
  vc_shape_t cs = *sh;
  cs.B = 1;
  cs.H = hc;
  RunHostLayout L;
  size_t off = 0;
  for (int slot = 0; slot < 2; ++slot) {
    for (int i = 0; i < 3; ++i) {
      L.in[slot][i] = off;
      off += align256(chunk_bytes);
    }
    L.out[slot] = off;
    off += align256(chunk_bytes);
  }
  L.prep_ws_bytes = ws_layout(&cs, cfg).total;
  L.planes_bytes = nv ? 2 * n * 128 * S_pad : 0;
  for (int slot = 0; slot < 2; ++slot) {
    L.perm[slot] = off;     off += align256(n * S * 4);
    L.mu[slot] = off;       off += align256(n * nb * 128 * 4);
    L.v_codes[slot] = off;  off += align256(n * 128 * (nv || mx ? S_pad / 2 : S_pad));
    L.v_scales[slot] = off; off += nv ? align256(n * 128 * (S_pad / 16)) : mx ? align256(n * nb * 128 * 4) : 0;
    L.s_v[slot] = off;      off += align256(n * 4 * (ch ? 128 : 1));
    L.q_codes[slot] = off;  off += align256(n * S_pad * 128);
    L.q_scales[slot] = off; off += align256(n * nb * 4);
    L.k_codes[slot] = off;  off += align256(n * S_pad * 128);
    L.k_scales[slot] = off; off += align256(n * nb * 4);
    L.prep_ws[slot] = off;  off += align256(L.prep_ws_bytes);
    L.planes[slot] = off;   off += align256(L.planes_bytes);
  }
  L.total = off;
  return L;
}

// The internal streams of a device (host to device copies, device to host
// copies, the compute of odd chunks), created on first use and kept until the
// process exits.
std::mutex g_copy_mu;
cudaStream_t g_copy_streams[64][3];

vc_status_t copy_streams(int dev, cudaStream_t* h2d, cudaStream_t* d2h, cudaStream_t* odd) {
  std::lock_guard<std::mutex> lk(g_copy_mu);
  for (int i = 0; i < 3; ++i)
    if (!g_copy_streams[dev][i]) {
      cudaError_t e = cudaStreamCreateWithFlags(&g_copy_streams[dev][i], cudaStreamNonBlocking);
      if (e != cudaSuccess) {
        g_copy_streams[dev][i] = nullptr;
        return cuda_fail(e, "creating an internal stream");
      }
    }
  *h2d = g_copy_streams[dev][0];
  *d2h = g_copy_streams[dev][1];
  *odd = g_copy_streams[dev][2];
  return VC_OK;
}

// Events of one call, destroyed when the call returns (the runtime releases an
// event whose recorded work is still pending once that work completes).
struct CallEvents {
  cudaEvent_t start = nullptr, done = nullptr, in[2] = {nullptr, nullptr}, comp[2] = {nullptr, nullptr},
              out[2] = {nullptr, nullptr};
  cudaError_t create() {
    cudaEvent_t* all[8] = {&start, &done, &in[0], &in[1], &comp[0], &comp[1], &out[0], &out[1]};
    for (cudaEvent_t* e : all) {
      cudaError_t r = cudaEventCreateWithFlags(e, cudaEventDisableTiming);
      if (r != cudaSuccess) return r;
    }
    return cudaSuccess;
  }
  ~CallEvents() {
    cudaEvent_t all[8] = {start, done, in[0], in[1], comp[0], comp[1], out[0], out[1]};
    for (cudaEvent_t e : all)
      if (e) cudaEventDestroy(e);
  }
};

}  // namespace

extern "C" {

size_t vc_attn_run_host_workspace_bytes(const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                                        int32_t head_chunk) {
  if (check_shape(shape) != VC_OK || check_cfg(cfg) != VC_OK || head_chunk < 1) return 0;
  return run_host_layout(shape, cfg, head_chunk < shape->H ? head_chunk : shape->H).total;
}

vc_status_t vc_attn_run_host(const void* q, const void* k, const void* v, const vc_shape_t* shape,
                             const vc_vsmooth_cfg_t* cfg, float softmax_scale, int32_t k_p, void* o,
                             int32_t head_chunk, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                             void* stream) {
  NvtxRange range("vc_attn_run_host");
  g_last_error.clear();
  vc_status_t st;
  if ((st = check_shape(shape)) != VC_OK) return st;
  if ((st = check_cfg(cfg)) != VC_OK) return st;
  if (!q || !k || !v || !o) return fail(VC_ERR_INVALID_ARG, "q, k, v and o must be non-NULL");
  if (head_chunk < 1) return fail(VC_ERR_INVALID_ARG, "head_chunk must be >= 1 (got %d)", head_chunk);
  if (!(softmax_scale > 0.0f) || !(softmax_scale < 1e30f))
    return fail(VC_ERR_INVALID_ARG, "softmax_scale must be positive and finite");
  if (k_p < 0 || k_p > 8) return fail(VC_ERR_INVALID_ARG, "k_p must be in [0, 8] (got %d)", k_p);
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u))
    return fail(VC_ERR_INVALID_ARG, "dev_status must be 4-byte aligned");
  const int B = shape->B, S = shape->S, H = shape->H;
  const int hc = head_chunk < H ? head_chunk : H;
  const RunHostLayout L = run_host_layout(shape, cfg, hc);
  if (!workspace || workspace_bytes < L.total)
    return fail(VC_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", L.total,
                workspace ? workspace_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VC_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((st = ensure_device()) != VC_OK) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  cudaStream_t s_in, s_out, s_odd;
  if ((st = copy_streams(dev, &s_in, &s_out, &s_odd)) != VC_OK) return st;
  CallEvents ev;
  if ((e = ev.create()) != cudaSuccess) return cuda_fail(e, "creating events");
  const cudaStream_t cs_stream = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool nv = cfg->residual_fmt == VC_RESIDUAL_NVFP4, mx = cfg->residual_fmt == VC_RESIDUAL_MXFP4;
  const FwdKind kind = nv ? FwdKind::NVFP4
                          : mx ? FwdKind::MXFP4
                               : cfg->residual_fmt == VC_RESIDUAL_E4M3_PER_CHANNEL ? FwdKind::E4M3_CHANNEL
                                                                                   : FwdKind::E4M3;
  const size_t row_bytes = (size_t)H * 256;  // one token of all heads
  const char* hq[3] = {static_cast<const char*>(q), static_cast<const char*>(k), static_cast<const char*>(v)};
  char* ho = static_cast<char*>(o);
  // the copies start after the work already on the caller's stream (it may still
  // be using the workspace)
  if ((e = cudaEventRecord(ev.start, cs_stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if ((e = cudaStreamWaitEvent(s_in, ev.start, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  if ((e = cudaStreamWaitEvent(s_out, ev.start, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  if ((e = cudaStreamWaitEvent(s_odd, ev.start, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  const cudaStream_t comp_stream[2] = {cs_stream, s_odd};
  // Chunks of hc heads of one batch entry; the first and the last chunk of the
  // call take a single head, so that the copy-in before the first compute and
  // the copy-out after the last one (neither overlaps anything) are short.
  std::vector<std::pair<int, int>> chunks;  // (b * H + h0, heads)
  for (int b = 0; b < B; ++b)
    for (int h0 = 0; h0 < H; h0 += hc) chunks.emplace_back(b * H + h0, hc < H - h0 ? hc : H - h0);
  if (chunks.front().second > 1) {
    chunks.front().second -= 1;
    chunks.front().first += 1;
    chunks.insert(chunks.begin(), std::make_pair(chunks.front().first - 1, 1));
  }
  if (chunks.size() > 1 && chunks.back().second > 1) {
    chunks.back().second -= 1;
    chunks.emplace_back(chunks.back().first + chunks.back().second, 1);
  }
  for (int c = 0; c < (int)chunks.size(); ++c) {
    {
      const int b = chunks[c].first / H, h0 = chunks[c].first % H, n = chunks[c].second, slot = c & 1;
      const size_t host_off = ((size_t)b * S * H + h0) * 256, crow = (size_t)n * 256;
      vc_shape_t cs = *shape;
      cs.B = 1;
      cs.H = n;
      // copy in (the slot's previous chunk must have been computed)
      if (c >= 2 && (e = cudaStreamWaitEvent(s_in, ev.comp[slot], 0)) != cudaSuccess)
        return cuda_fail(e, "cudaStreamWaitEvent");
      for (int i = 0; i < 3; ++i)
        if ((e = cudaMemcpy2DAsync(ws + L.in[slot][i], crow, hq[i] + host_off, row_bytes, crow, (size_t)S,
                                   cudaMemcpyHostToDevice, s_in)) != cudaSuccess)
          return cuda_fail(e, "copying an input chunk to the device");
      if ((e = cudaEventRecord(ev.in[slot], s_in)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
      // compute (the slot's previous output must have been copied out)
      const cudaStream_t cst = comp_stream[slot];
      if ((e = cudaStreamWaitEvent(cst, ev.in[slot], 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
      if (c >= 2 && (e = cudaStreamWaitEvent(cst, ev.out[slot], 0)) != cudaSuccess)
        return cuda_fail(e, "cudaStreamWaitEvent");
      vc_prepared_v_t pv;
      pv.perm = reinterpret_cast<int32_t*>(ws + L.perm[slot]);
      pv.mu = reinterpret_cast<float*>(ws + L.mu[slot]);
      pv.v_codes = ws + L.v_codes[slot];
      pv.v_scales = nv || mx ? ws + L.v_scales[slot] : nullptr;
      pv.s_v = reinterpret_cast<float*>(ws + L.s_v[slot]);
      vc_qk_fp8_t qk;
      qk.q_codes = ws + L.q_codes[slot];
      qk.q_scales = reinterpret_cast<float*>(ws + L.q_scales[slot]);
      qk.k_codes = ws + L.k_codes[slot];
      qk.k_scales = reinterpret_cast<float*>(ws + L.k_scales[slot]);
      if ((st = prepare_v_impl(ws + L.in[slot][2], &cs, cfg, &pv, ws + L.prep_ws[slot], L.prep_ws_bytes, nullptr,
                               cst, H, b, h0)) != VC_OK)
        return st;
      if ((st = vc_attn_quant_qk(ws + L.in[slot][0], ws + L.in[slot][1], &cs, pv.perm, &qk, cst)) != VC_OK)
        return st;
      if ((st = forward_common(&qk, &pv, &cs, softmax_scale, k_p, ws + L.out[slot], dev_status, cst, kind,
                               nv ? ws + L.planes[slot] : nullptr, L.planes_bytes)) != VC_OK)
        return st;
      if ((e = cudaEventRecord(ev.comp[slot], cst)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
      // copy out
      if ((e = cudaStreamWaitEvent(s_out, ev.comp[slot], 0)) != cudaSuccess)
        return cuda_fail(e, "cudaStreamWaitEvent");
      if ((e = cudaMemcpy2DAsync(ho + host_off, row_bytes, ws + L.out[slot], crow, crow, (size_t)S,
                                 cudaMemcpyDeviceToHost, s_out)) != cudaSuccess)
        return cuda_fail(e, "copying an output chunk to the host");
      if ((e = cudaEventRecord(ev.out[slot], s_out)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    }
  }
  // the caller's stream passes this point once the last output chunk is on the host
  if ((e = cudaEventRecord(ev.done, s_out)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if ((e = cudaStreamWaitEvent(cs_stream, ev.done, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  return VC_OK;
}

}  // extern "C"
