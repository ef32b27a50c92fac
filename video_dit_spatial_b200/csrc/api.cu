// C ABI of libsvg (declared in include/svg.h): argument validation, geometry,
// tensor-map encoding and the launches of the kernels in the other
// translation units. Every entry point validates everything on the host
// before it launches anything.
#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace svg {

// Status word of this module: device kernels OR error bits into it; the host
// passes its address to every kernel and reads it back in
// svg_get_device_status.
__device__ int g_device_status;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
int* g_status_ptr[kMaxDevices] = {};
void* g_status_ctx[kMaxDevices] = {};  // context the cached address belongs to
int g_is_sm100[kMaxDevices] = {};  // 0 unknown, 1 yes, -1 no

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn g_ctx_get = nullptr;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Driver entry points are looked up under a mutex of their own, which is never
// held while anything else is called.
std::mutex g_entry_mutex;

EncodeTiledFn encode_fn() {
  std::lock_guard<std::mutex> lock(g_entry_mutex);
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return g_encode;
}

CtxGetCurrentFn ctx_get_fn() {
  std::lock_guard<std::mutex> lock(g_entry_mutex);
  if (g_ctx_get == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get = reinterpret_cast<CtxGetCurrentFn>(fn);
  }
  return g_ctx_get;
}

inline bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

svg_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVG_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SVG_ERR_UNSUPPORTED;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_is_sm100[dev] != 0) return g_is_sm100[dev] > 0 ? SVG_OK : SVG_ERR_UNSUPPORTED;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SVG_ERR_CUDA;
  const bool ok = major == 10 && minor == 0;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_is_sm100[dev] = ok ? 1 : -1;
  return ok ? SVG_OK : SVG_ERR_UNSUPPORTED;
}

// Geometry checks shared by every entry point. `need_kernel_shape` also asks
// for the head dims / block sizes the kernels are built for.
svg_status check_geom(const svg_geom* g, bool need_kernel_shape) {
  if (g == nullptr) return SVG_ERR_INVALID_ARG;
  if (g->B < 1 || g->H < 1 || g->T < 1 || g->P < 1 || g->n_text < 0) return SVG_ERR_INVALID_ARG;
  if (g->spatial_band < 0 || g->temporal_width < 0) return SVG_ERR_INVALID_ARG;
  if (g->block_q < 1 || g->block_k < 1 || g->head_dim < 1) return SVG_ERR_INVALID_ARG;
  const int64_t N = static_cast<int64_t>(g->T) * g->P + g->n_text;
  if (N > (static_cast<int64_t>(1) << 30)) return SVG_ERR_INVALID_ARG;
  const int64_t BH = static_cast<int64_t>(g->B) * g->H;
  if (BH > 65535) return SVG_ERR_INVALID_ARG;
  if (!(g->scale > 0.0f) || !(g->scale < 3.0e38f)) return SVG_ERR_INVALID_ARG;
  if (need_kernel_shape) {
    if (g->head_dim != 64 && g->head_dim != 128) return SVG_ERR_UNSUPPORTED;
    if ((g->block_q != 64 && g->block_q != 128) || (g->block_k != 64 && g->block_k != 128))
      return SVG_ERR_UNSUPPORTED;
    const int64_t nqb = (N + g->block_q - 1) / g->block_q;
    if (nqb > 0x7fffffff) return SVG_ERR_INVALID_ARG;
  }
  return SVG_OK;
}

int64_t mask_nnz_host(const Dims& d, int32_t kind) {
  const MaskGeom m = make_mask_geom(d, kind);
  int64_t nnz = 0;
  for (int32_t r = 0; r < d.nqb; ++r) nnz += mask_row(m, r).count();
  return nnz;
}

}  // namespace

Dims make_dims(const svg_geom& g) {
  Dims d;
  d.B = g.B;
  d.H = g.H;
  d.BH = g.B * g.H;
  d.T = g.T;
  d.P = g.P;
  d.n_text = g.n_text;
  d.d = g.head_dim;
  d.bq = g.block_q;
  d.bk = g.block_k;
  d.s = g.spatial_band;
  d.w = g.temporal_width;
  d.Nv = g.T * g.P;
  d.N = d.Nv + g.n_text;
  d.nqb = (d.N + d.bq - 1) / d.bq;
  d.nkb = (d.N + d.bk - 1) / d.bk;
  d.scale = g.scale;
  return d;
}

void* current_context() {
  CtxGetCurrentFn get = ctx_get_fn();
  CUcontext c = nullptr;
  if (get == nullptr || get(&c) != CUDA_SUCCESS) return nullptr;
  return static_cast<void*>(c);
}

int* device_status_word(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  // A device reset tears the context down and the module is loaded again into
  // the next one, at a new address: look it up again whenever the context
  // changes. No lock is held while the runtime or the driver is called.
  void* ctx = current_context();
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_status_ptr[dev] != nullptr && ctx != nullptr && g_status_ctx[dev] == ctx)
      return g_status_ptr[dev];
  }
  void* ptr = nullptr;
  *err = cudaGetSymbolAddress(&ptr, g_device_status);  // initialises the context if needed
  if (*err != cudaSuccess) return nullptr;
  void* now = current_context();
  std::lock_guard<std::mutex> lock(g_mutex);
  g_status_ptr[dev] = static_cast<int*>(ptr);
  g_status_ctx[dev] = now;
  return g_status_ptr[dev];
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, int32_t d, int32_t N, int32_t BH,
                    int32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(d) * 2 * static_cast<cuuint64_t>(N)};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_u8_rows128(CUtensorMap* map, const void* base, int32_t N, int32_t BH,
                          int32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {128u, static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {128u, 128u * static_cast<cuuint64_t>(N)};
  const cuuint32_t box[3] = {128u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_rows_bf16(CUtensorMap* map, const void* base, int32_t d, int64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {64u, 1u};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace svg

using svg::Dims;

extern "C" {

const char* svg_status_string(svg_status s) {
  switch (s) {
    case SVG_OK: return "SVG_OK";
    case SVG_ERR_INVALID_ARG: return "SVG_ERR_INVALID_ARG";
    case SVG_ERR_UNSUPPORTED: return "SVG_ERR_UNSUPPORTED";
    case SVG_ERR_CAPACITY: return "SVG_ERR_CAPACITY";
    case SVG_ERR_CUDA: return "SVG_ERR_CUDA";
    case SVG_ERR_DEVICE_TIMEOUT: return "SVG_ERR_DEVICE_TIMEOUT";
  }
  return "SVG_ERR_UNKNOWN";
}

int32_t svg_version(void) { return 100; }

svg_status svg_mask_nnz(const svg_geom* geom, int32_t kind, int64_t* nnz) {
  if (nnz == nullptr) return SVG_ERR_INVALID_ARG;
  if (kind < SVG_MASK_SPATIAL || kind > SVG_MASK_DENSE) return SVG_ERR_INVALID_ARG;
  const svg_status st = svg::check_geom(geom, false);
  if (st != SVG_OK) return st;
  const Dims d = svg::make_dims(*geom);
  *nnz = svg::mask_nnz_host(d, kind);
  return SVG_OK;
}

svg_status svg_build_block_mask(const svg_geom* geom, int32_t kind, int32_t* row_ptr,
                                int32_t* col_idx, int64_t col_capacity, svg_stream_t stream) {
  if (row_ptr == nullptr || col_idx == nullptr) return SVG_ERR_INVALID_ARG;
  if (kind < SVG_MASK_SPATIAL || kind > SVG_MASK_DENSE) return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_geom(geom, false);
  if (st != SVG_OK) return st;
  const Dims d = svg::make_dims(*geom);
  const int64_t nnz = svg::mask_nnz_host(d, kind);
  if (nnz > 0x7fffffffLL) return SVG_ERR_INVALID_ARG;
  if (col_capacity < nnz) return SVG_ERR_CAPACITY;
  if ((st = svg::check_device()) != SVG_OK) return st;
  if (svg::launch_block_mask(d, kind, row_ptr, col_idx, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return SVG_ERR_CUDA;
  return SVG_OK;
}

svg_status svg_profile_workspace_bytes(const svg_geom* geom, int32_t n_samples, size_t* bytes) {
  if (bytes == nullptr || n_samples < 1) return SVG_ERR_INVALID_ARG;
  const svg_status st = svg::check_geom(geom, false);
  if (st != SVG_OK) return st;
  const Dims d = svg::make_dims(*geom);
  *bytes = svg::profile_workspace_bytes(d, n_samples, svg::profile_splits(d, n_samples));
  return SVG_OK;
}

svg_status svg_profile_heads(const svg_geom* geom, const svg_bf16* q, const svg_bf16* k,
                             const svg_bf16* v, const int32_t* sample_idx, int32_t n_samples,
                             int8_t* labels, float* mse, void* workspace, size_t workspace_bytes,
                             svg_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || sample_idx == nullptr ||
      labels == nullptr || workspace == nullptr)
    return SVG_ERR_INVALID_ARG;
  if (!svg::aligned16(q) || !svg::aligned16(k) || !svg::aligned16(v)) return SVG_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_geom(geom, true);
  if (st != SVG_OK) return st;
  const Dims d = svg::make_dims(*geom);
  if (n_samples < 1 || n_samples > d.Nv) return SVG_ERR_INVALID_ARG;
  size_t need = 0;
  svg_profile_workspace_bytes(geom, n_samples, &need);
  if (workspace_bytes < need) return SVG_ERR_CAPACITY;
  if ((st = svg::check_device()) != SVG_OK) return st;
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  svg::ProfileArgs a{q,      k,   v, sample_idx, n_samples, labels, mse, static_cast<float*>(workspace),
                     svg::profile_splits(d, n_samples)};
  if (svg::launch_profile(d, a, status, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SVG_ERR_CUDA;
  return SVG_OK;
}

svg_status svg_profile_heads_noalloc(const svg_geom* geom, const svg_bf16* q, const svg_bf16* k,
                                     const svg_bf16* v, const int32_t* sample_idx,
                                     int32_t n_samples, int8_t* labels, float* mse,
                                     svg_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || sample_idx == nullptr || labels == nullptr)
    return SVG_ERR_INVALID_ARG;
  if (!svg::aligned16(q) || !svg::aligned16(k) || !svg::aligned16(v)) return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_geom(geom, true);
  if (st != SVG_OK) return st;
  const Dims d = svg::make_dims(*geom);
  if (n_samples < 1 || n_samples > d.Nv) return SVG_ERR_INVALID_ARG;
  // one key range per (head, sample tile): only the per-tile errors
  const size_t need = svg::profile_workspace_bytes(d, n_samples, 1);
  if (need > svg::profile_noalloc_scratch_bytes()) return SVG_ERR_CAPACITY;
  if ((st = svg::check_device()) != SVG_OK) return st;
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  svg::ProfileArgs a{q, k, v, sample_idx, n_samples, labels, mse, nullptr, 1};
  if (svg::launch_profile_noalloc(d, a, status, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SVG_ERR_CUDA;
  return SVG_OK;
}

static svg_status permute_common(const svg_geom* geom, int n, const svg_bf16* const* in,
                                 svg_bf16* const* out, const int8_t* labels, bool inverse,
                                 svg_stream_t stream) {
  svg_status st = svg::check_geom(geom, false);
  if (st != SVG_OK) return st;
  if (geom->head_dim != 64 && geom->head_dim != 128) return SVG_ERR_UNSUPPORTED;
  const Dims d = svg::make_dims(*geom);
  const size_t bytes = static_cast<size_t>(d.BH) * d.N * d.d * 2;
  for (int t = 0; t < n; ++t) {
    if (in[t] == nullptr || out[t] == nullptr) return SVG_ERR_INVALID_ARG;
    if (!svg::aligned16(in[t]) || !svg::aligned16(out[t])) return SVG_ERR_INVALID_ARG;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(in[t]), b0 = reinterpret_cast<uintptr_t>(out[t]);
    if (a0 < b0 + bytes && b0 < a0 + bytes) return SVG_ERR_INVALID_ARG;  // overlap
  }
  if ((st = svg::check_device()) != SVG_OK) return st;
  if (svg::launch_permute(d, n, in, out, labels, inverse, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return SVG_ERR_CUDA;
  return SVG_OK;
}

svg_status svg_permute(const svg_geom* geom, const svg_bf16* in, svg_bf16* out,
                       const int8_t* labels, svg_stream_t stream) {
  const svg_bf16* i[1] = {in};
  svg_bf16* o[1] = {out};
  return permute_common(geom, 1, i, o, labels, false, stream);
}

svg_status svg_unpermute(const svg_geom* geom, const svg_bf16* in, svg_bf16* out,
                         const int8_t* labels, svg_stream_t stream) {
  const svg_bf16* i[1] = {in};
  svg_bf16* o[1] = {out};
  return permute_common(geom, 1, i, o, labels, true, stream);
}

svg_status svg_permute_qkv(const svg_geom* geom, const svg_bf16* q, const svg_bf16* k,
                           const svg_bf16* v, svg_bf16* qp, svg_bf16* kp, svg_bf16* vp,
                           const int8_t* labels, svg_stream_t stream) {
  if ((q == nullptr) != (qp == nullptr)) return SVG_ERR_INVALID_ARG;
  if (q == nullptr) {  // K and V only
    const svg_bf16* i[2] = {k, v};
    svg_bf16* o[2] = {kp, vp};
    return permute_common(geom, 2, i, o, labels, false, stream);
  }
  const svg_bf16* i[3] = {q, k, v};
  svg_bf16* o[3] = {qp, kp, vp};
  return permute_common(geom, 3, i, o, labels, false, stream);
}

svg_status svg_sparse_attention(const svg_geom* geom, const svg_bf16* q, const svg_bf16* k,
                                const svg_bf16* v, const svg_bf16* qp, const svg_bf16* kp,
                                const svg_bf16* vp, const int8_t* labels,
                                const int32_t* row_ptr_s, const int32_t* col_idx_s,
                                const int32_t* row_ptr_t, const int32_t* col_idx_t, svg_bf16* o,
                                svg_bf16* op, float* lse, svg_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || row_ptr_s == nullptr ||
      col_idx_s == nullptr)
    return SVG_ERR_INVALID_ARG;
  const bool any_perm = qp || kp || vp || op;
  const bool all_perm = qp && kp && vp && op;
  if (any_perm && !all_perm) return SVG_ERR_INVALID_ARG;
  if (all_perm && (row_ptr_t == nullptr || col_idx_t == nullptr)) return SVG_ERR_INVALID_ARG;
  const svg_bf16* tensors[8] = {q, k, v, o, qp, kp, vp, op};
  for (int t = 0; t < 8; ++t)
    if (tensors[t] != nullptr && !svg::aligned16(tensors[t])) return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_geom(geom, true);
  if (st != SVG_OK) return st;
  if ((st = svg::check_device()) != SVG_OK) return st;
  const Dims d = svg::make_dims(*geom);
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  svg::AttnArgs a{q, k, v, qp, kp, vp, labels, row_ptr_s, col_idx_s, row_ptr_t, col_idx_t,
                  o, op, lse, false, nullptr, nullptr};
  if (svg::launch_sparse_attention(d, a, status, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return SVG_ERR_CUDA;
  return SVG_OK;
}

svg_status svg_quantize_v_e4m3(const svg_geom* geom, const svg_bf16* v, const svg_bf16* vp,
                               const int8_t* labels, uint8_t* v8, float* v_scale,
                               svg_stream_t stream) {
  if (v == nullptr || v8 == nullptr || v_scale == nullptr) return SVG_ERR_INVALID_ARG;
  if (labels != nullptr && vp == nullptr) return SVG_ERR_INVALID_ARG;
  if (!svg::aligned16(v) || !svg::aligned16(v8) || (vp != nullptr && !svg::aligned16(vp)) ||
      (reinterpret_cast<uintptr_t>(v_scale) & 3u) != 0)
    return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_geom(geom, false);
  if (st != SVG_OK) return st;
  if (geom->head_dim != 128) return SVG_ERR_UNSUPPORTED;
  if ((st = svg::check_device()) != SVG_OK) return st;
  const Dims d = svg::make_dims(*geom);
  return svg::launch_quantize_v(d, v, vp, labels, v8, v_scale,
                                static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SVG_OK
             : SVG_ERR_CUDA;
}

svg_status svg_sparse_attention_fp8pv(const svg_geom* geom, const svg_bf16* q, const svg_bf16* k,
                                      const svg_bf16* qp, const svg_bf16* kp, const uint8_t* v8,
                                      const float* v_scale, const int8_t* labels,
                                      const int32_t* row_ptr_s, const int32_t* col_idx_s,
                                      const int32_t* row_ptr_t, const int32_t* col_idx_t,
                                      svg_bf16* o, svg_bf16* op, float* lse,
                                      svg_stream_t stream) {
  if (q == nullptr || k == nullptr || v8 == nullptr || v_scale == nullptr || o == nullptr ||
      row_ptr_s == nullptr || col_idx_s == nullptr)
    return SVG_ERR_INVALID_ARG;
  const bool any_perm = qp || kp || op;
  const bool all_perm = qp && kp && op;
  if (any_perm && !all_perm) return SVG_ERR_INVALID_ARG;
  if (all_perm && (row_ptr_t == nullptr || col_idx_t == nullptr)) return SVG_ERR_INVALID_ARG;
  const void* tensors[6] = {q, k, o, qp, kp, op};
  for (int t = 0; t < 6; ++t)
    if (tensors[t] != nullptr && !svg::aligned16(tensors[t])) return SVG_ERR_INVALID_ARG;
  if (!svg::aligned16(v8) || (reinterpret_cast<uintptr_t>(v_scale) & 3u) != 0)
    return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_geom(geom, true);
  if (st != SVG_OK) return st;
  if (geom->head_dim != 128 || geom->block_q != 128) return SVG_ERR_UNSUPPORTED;
  if ((st = svg::check_device()) != SVG_OK) return st;
  const Dims d = svg::make_dims(*geom);
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  svg::AttnArgs a{q, k, nullptr, qp, kp, nullptr, labels, row_ptr_s, col_idx_s, row_ptr_t,
                  col_idx_t, o, op, lse, false, v8, v_scale};
  err = svg::launch_sparse_attention(d, a, status, static_cast<cudaStream_t>(stream));
  if (err == cudaErrorNotSupported) return SVG_ERR_UNSUPPORTED;
  return err == cudaSuccess ? SVG_OK : SVG_ERR_CUDA;
}

svg_status svg_sparse_attention_fused(const svg_geom* geom, const svg_bf16* q,
                                      const svg_bf16* k, const svg_bf16* v,
                                      const svg_bf16* kp, const svg_bf16* vp,
                                      const int8_t* labels, const int32_t* row_ptr_s,
                                      const int32_t* col_idx_s, const int32_t* row_ptr_t,
                                      const int32_t* col_idx_t, svg_bf16* o, float* lse,
                                      svg_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || labels == nullptr ||
      row_ptr_s == nullptr || col_idx_s == nullptr || row_ptr_t == nullptr ||
      col_idx_t == nullptr)
    return SVG_ERR_INVALID_ARG;
  if (!svg::aligned16(q) || !svg::aligned16(k) || !svg::aligned16(v) || !svg::aligned16(o))
    return SVG_ERR_INVALID_ARG;
  if ((kp == nullptr) != (vp == nullptr)) return SVG_ERR_INVALID_ARG;
  if (kp != nullptr && (!svg::aligned16(kp) || !svg::aligned16(vp))) return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_geom(geom, true);
  if (st != SVG_OK) return st;
  if (geom->block_q != 128) return SVG_ERR_UNSUPPORTED;
  // gather coordinates are signed 32-bit rows of the [B*H*N, d] view
  const int64_t rows = static_cast<int64_t>(geom->B) * geom->H *
                       (static_cast<int64_t>(geom->T) * geom->P + geom->n_text);
  if (rows > 0x7fffffffLL) return SVG_ERR_UNSUPPORTED;
  if ((st = svg::check_device()) != SVG_OK) return st;
  const Dims d = svg::make_dims(*geom);
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  svg::AttnArgs a{q, k, v, nullptr, kp, vp, labels, row_ptr_s, col_idx_s,
                  row_ptr_t, col_idx_t, o, nullptr, lse, true, nullptr, nullptr};
  err = svg::launch_sparse_attention(d, a, status, static_cast<cudaStream_t>(stream));
  if (err == cudaErrorNotSupported) return SVG_ERR_UNSUPPORTED;
  return err == cudaSuccess ? SVG_OK : SVG_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// semantic-aware permutation (Sparse VideoGen 2)
// ---------------------------------------------------------------------------
static svg_status check_kmeans_shape(int32_t BH, int32_t N, int32_t d, int32_t C) {
  if (BH < 1 || BH > 65535 || N < 1 || N > (1 << 30)) return SVG_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SVG_ERR_UNSUPPORTED;
  if (C < 16 || C > 256 || C % 16 != 0) return SVG_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(BH) * N > 0x7fffffffLL) return SVG_ERR_INVALID_ARG;
  return SVG_OK;
}

svg_status svg2_kmeans_workspace_bytes(int32_t BH, int32_t N, int32_t d, int32_t C,
                                       size_t* bytes) {
  if (bytes == nullptr) return SVG_ERR_INVALID_ARG;
  const svg_status st = check_kmeans_shape(BH, N, d, C);
  if (st != SVG_OK) return st;
  *bytes = svg::kmeans_workspace_bytes(BH, N, d, C);
  return SVG_OK;
}

static svg_status kmeans_common(int32_t BH, int32_t N, int32_t d, int32_t C, const svg_bf16* x,
                                const float* c_in, float* c_out, int32_t* assign, int32_t* order,
                                int32_t* offsets, void* ws, size_t ws_bytes, int** status) {
  if (x == nullptr || c_out == nullptr || assign == nullptr || order == nullptr ||
      offsets == nullptr || ws == nullptr)
    return SVG_ERR_INVALID_ARG;
  svg_status st = check_kmeans_shape(BH, N, d, C);
  if (st != SVG_OK) return st;
  if (!svg::aligned16(x) || !svg::aligned16(c_out) || (c_in && !svg::aligned16(c_in)) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 ||
      (reinterpret_cast<uintptr_t>(assign) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(order) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(offsets) & 3u) != 0)
    return SVG_ERR_INVALID_ARG;
  if (ws_bytes < svg::kmeans_workspace_bytes(BH, N, d, C)) return SVG_ERR_CAPACITY;
  if ((st = svg::check_device()) != SVG_OK) return st;
  cudaError_t err;
  *status = svg::device_status_word(&err);
  return *status == nullptr ? SVG_ERR_CUDA : SVG_OK;
}

svg_status svg2_kmeans(int32_t BH, int32_t N, int32_t d, int32_t C, int32_t iters,
                       const svg_bf16* x, float* centroids, int32_t* assign, int32_t* order,
                       int32_t* offsets, void* workspace, size_t workspace_bytes,
                       svg_stream_t stream) {
  if (iters < 0 || iters > 1000) return SVG_ERR_INVALID_ARG;
  int* status = nullptr;
  const svg_status st = kmeans_common(BH, N, d, C, x, nullptr, centroids, assign, order, offsets,
                                      workspace, workspace_bytes, &status);
  if (st != SVG_OK) return st;
  return svg::launch_kmeans(BH, N, d, C, iters, x, centroids, assign, order, offsets, workspace,
                            status, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SVG_OK
             : SVG_ERR_CUDA;
}

svg_status svg2_kmeans_step(int32_t BH, int32_t N, int32_t d, int32_t C, const svg_bf16* x,
                            const float* centroids_in, float* centroids_out, int32_t* assign,
                            int32_t* order, int32_t* offsets, void* workspace,
                            size_t workspace_bytes, svg_stream_t stream) {
  if (centroids_in == nullptr || centroids_in == centroids_out) return SVG_ERR_INVALID_ARG;
  int* status = nullptr;
  const svg_status st = kmeans_common(BH, N, d, C, x, centroids_in, centroids_out, assign, order,
                                      offsets, workspace, workspace_bytes, &status);
  if (st != SVG_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (svg::launch_kmeans_assign(BH, N, d, C, x, centroids_in, assign, workspace, status, s) !=
          cudaSuccess ||
      svg::launch_cluster_sort(BH, N, C, assign, order, offsets, workspace, d, status, s) !=
          cudaSuccess ||
      svg::launch_kmeans_update(BH, N, d, C, x, order, offsets, centroids_in, centroids_out,
                                workspace, status, s) !=
          cudaSuccess)
    return SVG_ERR_CUDA;
  return SVG_OK;
}

svg_status svg2_select_clusters(int32_t BH, int32_t d, int32_t Cq, int32_t Ck, float scale,
                                float top_p, const float* cq, const float* ck,
                                const int32_t* offsets_k, const float* disp, float tau,
                                uint32_t* sel, svg_stream_t stream) {
  if (cq == nullptr || ck == nullptr || offsets_k == nullptr || sel == nullptr)
    return SVG_ERR_INVALID_ARG;
  if (BH < 1 || BH > 65535 || d < 1 || d > 4096 || Cq < 1 || Cq > 65535 || Ck < 1 || Ck > 1024)
    return SVG_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !(scale < 3.0e38f) || !(top_p > 0.0f) || !(top_p <= 1.0f))
    return SVG_ERR_INVALID_ARG;
  if (disp != nullptr && !(tau >= 0.0f)) return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_device();
  if (st != SVG_OK) return st;
  return svg::launch_select_clusters(BH, d, Cq, Ck, scale, top_p, cq, ck, offsets_k, disp, tau,
                                     sel, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SVG_OK
             : SVG_ERR_CUDA;
}

svg_status svg2_cluster_value_stats(int32_t BH, int32_t N, int32_t d, int32_t Ck,
                                    const svg_bf16* v, const int32_t* order_k,
                                    const int32_t* offsets_k, float* vbar, float* disp,
                                    svg_stream_t stream) {
  if (v == nullptr || order_k == nullptr || offsets_k == nullptr || vbar == nullptr ||
      disp == nullptr)
    return SVG_ERR_INVALID_ARG;
  if (BH < 1 || BH > 65535 || N < 1 || Ck < 1 || static_cast<int64_t>(BH) * N > 0x7fffffffLL)
    return SVG_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SVG_ERR_UNSUPPORTED;
  if (!svg::aligned16(v) || (reinterpret_cast<uintptr_t>(vbar) & 15u) != 0)
    return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_device();
  if (st != SVG_OK) return st;
  return svg::launch_cluster_stats(BH, N, d, Ck, v, order_k, offsets_k, vbar, disp,
                                   static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SVG_OK
             : SVG_ERR_CUDA;
}

svg_status svg2_ear_workspace_bytes(int32_t BH, int32_t d, int32_t Ck, size_t* bytes) {
  if (bytes == nullptr || BH < 1 || Ck < 1) return SVG_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SVG_ERR_UNSUPPORTED;
  *bytes = svg::ear_workspace_bytes(BH, d, Ck);
  return SVG_OK;
}

svg_status svg2_ear_compensate(int32_t BH, int32_t N, int32_t d, int32_t Ck, int32_t block_k,
                               float scale, const svg_bf16* qs, const float* kbar,
                               const float* vbar, const int32_t* offsets_k,
                               const int32_t* row_ptr, const int32_t* col_idx, svg_bf16* os,
                               const float* lse, void* workspace, size_t workspace_bytes,
                               svg_stream_t stream) {
  if (qs == nullptr || kbar == nullptr || vbar == nullptr || offsets_k == nullptr ||
      row_ptr == nullptr || col_idx == nullptr || os == nullptr || lse == nullptr ||
      workspace == nullptr)
    return SVG_ERR_INVALID_ARG;
  if (BH < 1 || BH > 65535 || N < 1 || N > (1 << 30)) return SVG_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SVG_ERR_UNSUPPORTED;
  if (Ck < 16 || Ck > 256 || Ck % 16 != 0) return SVG_ERR_UNSUPPORTED;
  if (block_k != 64 && block_k != 128) return SVG_ERR_UNSUPPORTED;
  if ((N + block_k - 1) / block_k > 4096) return SVG_ERR_UNSUPPORTED;
  if (!(scale > 0.0f) || !(scale < 3.0e38f)) return SVG_ERR_INVALID_ARG;
  if (!svg::aligned16(qs) || !svg::aligned16(os) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SVG_ERR_INVALID_ARG;
  if (workspace_bytes < svg::ear_workspace_bytes(BH, d, Ck)) return SVG_ERR_CAPACITY;
  svg_status st = svg::check_device();
  if (st != SVG_OK) return st;
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  return svg::launch_ear_compensate(BH, N, d, Ck, block_k, scale, qs, kbar, vbar, offsets_k,
                                    row_ptr, col_idx, os, lse, workspace, status,
                                    static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SVG_OK
             : SVG_ERR_CUDA;
}

svg_status svg2_build_tile_csr(int32_t BH, int32_t N, int32_t Cq, int32_t Ck, int32_t block_q,
                               int32_t block_k, const int32_t* offsets_q, const int32_t* offsets_k,
                               const uint32_t* sel, int32_t* row_ptr, int32_t* col_idx,
                               int64_t col_capacity, int32_t* counts, svg_stream_t stream) {
  if (offsets_q == nullptr || offsets_k == nullptr || sel == nullptr || row_ptr == nullptr ||
      col_idx == nullptr || counts == nullptr || col_capacity < 0)
    return SVG_ERR_INVALID_ARG;
  if (BH < 1 || BH > 65535 || N < 1 || N > (1 << 30) || Cq < 1 || Ck < 1 || Ck > 1024)
    return SVG_ERR_INVALID_ARG;
  if ((block_q != 64 && block_q != 128) || (block_k != 64 && block_k != 128))
    return SVG_ERR_UNSUPPORTED;
  const int64_t nqb = (N + block_q - 1) / block_q, nkb = (N + block_k - 1) / block_k;
  if (nkb > 4096) return SVG_ERR_UNSUPPORTED;
  if (BH * nqb > 0x7fffffffLL / 2) return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_device();
  if (st != SVG_OK) return st;
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  return svg::launch_tile_csr(BH, N, Cq, Ck, block_q, block_k, offsets_q, offsets_k, sel, row_ptr,
                              col_idx, col_capacity, counts, status,
                              static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SVG_OK
             : SVG_ERR_CUDA;
}

static svg_status rows_common(int32_t BH, int32_t N, int32_t d, const svg_bf16* x,
                              const int32_t* order, svg_bf16* y, bool scatter,
                              svg_stream_t stream) {
  if (x == nullptr || order == nullptr || y == nullptr) return SVG_ERR_INVALID_ARG;
  if (BH < 1 || N < 1 || static_cast<int64_t>(BH) * N > 0x7fffffffLL) return SVG_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SVG_ERR_UNSUPPORTED;
  if (!svg::aligned16(x) || !svg::aligned16(y)) return SVG_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(BH) * N * d * 2;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(x), b0 = reinterpret_cast<uintptr_t>(y);
  if (a0 < b0 + bytes && b0 < a0 + bytes) return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_device();
  if (st != SVG_OK) return st;
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  return svg::launch_permute_rows(BH, N, d, x, order, y, scatter, status,
                                  static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SVG_OK
             : SVG_ERR_CUDA;
}

svg_status svg2_gather_rows(int32_t BH, int32_t N, int32_t d, const svg_bf16* x,
                            const int32_t* order, svg_bf16* y, svg_stream_t stream) {
  return rows_common(BH, N, d, x, order, y, false, stream);
}

svg_status svg2_scatter_rows(int32_t BH, int32_t N, int32_t d, const svg_bf16* y_sorted,
                             const int32_t* order, svg_bf16* y, svg_stream_t stream) {
  return rows_common(BH, N, d, y_sorted, order, y, true, stream);
}

svg_status svg2_sparse_attention(int32_t BH, int32_t N, int32_t d, int32_t block_k, float scale,
                                 const svg_bf16* qs, const svg_bf16* ks, const svg_bf16* vs,
                                 const int32_t* row_ptr, const int32_t* col_idx, svg_bf16* os,
                                 float* lse, svg_stream_t stream) {
  if (qs == nullptr || ks == nullptr || vs == nullptr || row_ptr == nullptr ||
      col_idx == nullptr || os == nullptr)
    return SVG_ERR_INVALID_ARG;
  if (!svg::aligned16(qs) || !svg::aligned16(ks) || !svg::aligned16(vs) || !svg::aligned16(os))
    return SVG_ERR_INVALID_ARG;
  if (BH < 1 || BH > 65535 || N < 1 || N > (1 << 30)) return SVG_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !(scale < 3.0e38f)) return SVG_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || (block_k != 64 && block_k != 128)) return SVG_ERR_UNSUPPORTED;
  svg_status st = svg::check_device();
  if (st != SVG_OK) return st;
  // the sorted layouts are one sequence of N tokens per head, no text part
  svg_geom g{1, BH, 1, N, 0, d, 128, block_k, 0, 0, scale};
  const Dims dm = svg::make_dims(g);
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  svg::AttnArgs a{qs, ks, vs, nullptr, nullptr, nullptr, nullptr, row_ptr, col_idx, nullptr,
                  nullptr, os, nullptr, lse, false, nullptr, nullptr, true};
  err = svg::launch_sparse_attention(dm, a, status, static_cast<cudaStream_t>(stream));
  if (err == cudaErrorNotSupported) return SVG_ERR_UNSUPPORTED;
  return err == cudaSuccess ? SVG_OK : SVG_ERR_CUDA;
}

svg_status svg_get_device_status(svg_stream_t stream, int32_t* bits) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SVG_ERR_CUDA;
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  int value = 0;
  if (cudaMemcpyFromSymbol(&value, svg::g_device_status, sizeof(int)) != cudaSuccess)
    return SVG_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(svg::g_device_status, &zero, sizeof(int)) != cudaSuccess)
    return SVG_ERR_CUDA;
  if (bits != nullptr) *bits = value;
  if (value & svg::kDevErrTimeout) return SVG_ERR_DEVICE_TIMEOUT;
  if (value & svg::kDevErrBounds) return SVG_ERR_INVALID_ARG;
  return SVG_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- self-test
namespace svg {
namespace {
__global__ void wait_selftest_kernel(long long limit, int* status) {
  __shared__ uint64_t never;
  if (threadIdx.x == 0) {
    mbar_init(&never, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Same loop shape as mbar_wait, with a caller-chosen limit.
    const long long t0 = clock64();
    while (!mbar_try_wait(&never, 0)) {
      if (clock64() - t0 > limit) {
        atomicOr(status, kDevErrTimeout);
        break;
      }
    }
  }
  __syncthreads();
}
}  // namespace

cudaError_t launch_wait_selftest(long long limit_cycles, int* status, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_cycles, status);
  return cudaGetLastError();
}
}  // namespace svg

extern "C" svg_status svg_selftest_wait_timeout(int64_t limit_cycles, svg_stream_t stream) {
  if (limit_cycles < 1 || limit_cycles > (static_cast<int64_t>(1) << 31)) return SVG_ERR_INVALID_ARG;
  svg_status st = svg::check_device();
  if (st != SVG_OK) return st;
  cudaError_t err;
  int* status = svg::device_status_word(&err);
  if (status == nullptr) return SVG_ERR_CUDA;
  if (svg::launch_wait_selftest(limit_cycles, status, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return SVG_ERR_CUDA;
  return SVG_OK;
}
