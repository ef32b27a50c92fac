// Host-side declarations shared by the translation units of libsvg.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "svg.h"

namespace svg {

// Derived sizes of a validated geometry.
struct Dims {
  int32_t B, H, BH, T, P, n_text, d, bq, bk, s, w;
  int32_t N, Nv, nqb, nkb;
  float scale;
};

Dims make_dims(const svg_geom& g);

// Closed-form CSR row of a block mask: the key blocks of row r are the run
// [c_lo, c_hi] (empty when c_lo > c_hi) followed by the run [t_lo, t_hi]
// (empty when t_lo > t_hi), the second starting after the first. Shared by the
// host nnz count and the device builder so both agree by construction.
struct MaskRow {
  int32_t c_lo, c_hi, t_lo, t_hi;
  __host__ __device__ int32_t count() const {
    int32_t n = 0;
    if (c_hi >= c_lo) n += c_hi - c_lo + 1;
    if (t_hi >= t_lo) n += t_hi - t_lo + 1;
    return n;
  }
  __host__ __device__ int32_t at(int32_t k) const {
    const int32_t n1 = (c_hi >= c_lo) ? (c_hi - c_lo + 1) : 0;
    return k < n1 ? c_lo + k : t_lo + (k - n1);
  }
};

struct MaskGeom {
  int32_t N, Nv, bq, bk, nkb;
  int32_t group;   // tokens per group in the layout: P (spatial), T (temporal)
  int32_t ngroups; // number of groups: T (spatial), P (temporal)
  int32_t band;    // s (spatial) or w (temporal)
  int32_t dense;   // 1: every block is on
};

__host__ __device__ inline MaskRow mask_row(const MaskGeom& m, int32_t r) {
  MaskRow out;
  const int32_t lo = r * m.bq;
  const int32_t hi = (lo + m.bq < m.N) ? lo + m.bq : m.N;  // exclusive
  const bool row_text = hi > m.Nv;
  const int32_t text_first = m.Nv / m.bk;  // key block holding the first text token
  if (m.dense || row_text) {
    out.c_lo = 0;
    out.c_hi = m.nkb - 1;
    out.t_lo = 1;
    out.t_hi = 0;
    return out;
  }
  // Video-only query block: its groups form the interval [g_lo, g_hi].
  const int32_t g_lo = lo / m.group;
  const int32_t g_hi = (hi - 1) / m.group;
  const int32_t a = (g_lo - m.band > 0) ? g_lo - m.band : 0;
  const int64_t z64 = static_cast<int64_t>(g_hi) + m.band;
  const int32_t z = (z64 < m.ngroups - 1) ? static_cast<int32_t>(z64) : m.ngroups - 1;
  const int64_t first_key = static_cast<int64_t>(a) * m.group;
  int64_t last_key = static_cast<int64_t>(z + 1) * m.group - 1;
  if (last_key > m.Nv - 1) last_key = m.Nv - 1;
  out.c_lo = static_cast<int32_t>(first_key / m.bk);
  out.c_hi = static_cast<int32_t>(last_key / m.bk);
  if (m.N > m.Nv) {
    out.t_lo = (text_first > out.c_hi) ? text_first : out.c_hi + 1;
    out.t_hi = m.nkb - 1;
  } else {
    out.t_lo = 1;
    out.t_hi = 0;
  }
  return out;
}

MaskGeom make_mask_geom(const Dims& d, int32_t kind);

// Device address of this module's status word on the current device.
int* device_status_word(cudaError_t* err);
// Identity of the calling thread's current CUDA context, or NULL when none is
// current yet (the runtime makes the device's primary context current on its
// first call that needs one).
void* current_context();

// Tensor map of a [BH, N, d] bf16 tensor with a (64 x rows x 1) box, 128-byte swizzle.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int32_t d, int32_t N, int32_t BH,
                    int32_t box_rows);
// Tensor map of a [BH, N, 128] 8-bit tensor with a (128 x rows x 1) box (one
// 128-byte row per token), 128-byte swizzle.
bool make_tmap_u8_rows128(CUtensorMap* map, const void* base, int32_t N, int32_t BH,
                          int32_t box_rows);
// Row map of the same tensor seen as [BH*N, d] with a 64 x 1 box, 128-byte
// swizzle: the tensor map of tile::gather4 row gathers.
bool make_tmap_rows_bf16(CUtensorMap* map, const void* base, int32_t d, int64_t rows);

// Launchers (validated arguments; return the launch error).
cudaError_t launch_permute(const Dims& d, int n_tensors, const svg_bf16* const* in,
                           svg_bf16* const* out, const int8_t* labels, bool inverse,
                           cudaStream_t stream);
cudaError_t launch_block_mask(const Dims& d, int32_t kind, int32_t* row_ptr, int32_t* col_idx,
                              cudaStream_t stream);

struct AttnArgs {
  const svg_bf16 *q, *k, *v, *qp, *kp, *vp;
  const int8_t* labels;
  const int32_t *row_ptr_s, *col_idx_s, *row_ptr_t, *col_idx_t;
  svg_bf16 *o, *op;
  float* lse;
  bool fused;  // temporal heads gather from q, k, v and scatter to o (qp..op unused)
  // FP8 PV (v and vp unused): e4m3 V of every head in its own layout and the
  // per-(head, channel) scales, as written by svg_quantize_v_e4m3
  const uint8_t* v8;
  const float* v_scale;
  // one CSR per (b, h): row b*H*nQB + h*nQB + r, i.e. (bh * nQB + r)
  bool csr_per_head = false;
};
cudaError_t launch_sparse_attention(const Dims& d, const AttnArgs& a, int* status,
                                    cudaStream_t stream);

struct ProfileArgs {
  const svg_bf16 *q, *k, *v;
  const int32_t* sample_idx;
  int32_t n_samples;
  int8_t* labels;
  float* mse;
  float* partial;    // the workspace: [BH][2][n_tiles] errors, then the split partials
  int32_t n_splits;  // key-range splits per (head, sample tile), profile_splits()
};
int32_t profile_tiles(int32_t n_samples);
int32_t profile_splits(const Dims& d, int32_t n_samples);
size_t profile_workspace_bytes(const Dims& d, int32_t n_samples, int32_t n_splits);
cudaError_t launch_profile(const Dims& d, const ProfileArgs& a, int* status, cudaStream_t stream);
// Same launch with the partial sums in the module's fixed device scratch
// (a.partial is ignored); see svg_profile_heads_noalloc.
size_t profile_noalloc_scratch_bytes();
cudaError_t launch_profile_noalloc(const Dims& d, const ProfileArgs& a, int* status,
                                   cudaStream_t stream);

// e4m3 quantisation of V (each head read from v or, if labelled temporal, vp):
// amax per (head, channel) into v_scale, the codes into v8, then v_scale
// turned into the dequantisation scale amax / 448.
cudaError_t launch_quantize_v(const Dims& d, const svg_bf16* v, const svg_bf16* vp,
                              const int8_t* labels, uint8_t* v8, float* v_scale,
                              cudaStream_t stream);

// Semantic-aware permutation (svg2.cu).
size_t kmeans_workspace_bytes(int32_t BH, int32_t N, int32_t D, int32_t C);
cudaError_t launch_kmeans(int32_t BH, int32_t N, int32_t D, int32_t C, int32_t iters,
                          const svg_bf16* x, float* centroids, int32_t* assign, int32_t* order,
                          int32_t* offsets, void* ws, int* status, cudaStream_t stream);
cudaError_t launch_kmeans_assign(int32_t BH, int32_t N, int32_t D, int32_t C, const svg_bf16* x,
                                 const float* centroids, int32_t* assign, void* ws, int* status,
                                 cudaStream_t stream);
cudaError_t launch_cluster_sort(int32_t BH, int32_t N, int32_t C, const int32_t* assign,
                                int32_t* order, int32_t* offsets, void* ws, int32_t D, int* status,
                                cudaStream_t stream);
cudaError_t launch_kmeans_update(int32_t BH, int32_t N, int32_t D, int32_t C, const svg_bf16* x,
                                 const int32_t* order, const int32_t* offsets, const float* c_in,
                                 float* c_out, void* ws, int* status, cudaStream_t stream);
cudaError_t launch_select_clusters(int32_t BH, int32_t D, int32_t Cq, int32_t Ck, float scale,
                                   float top_p, const float* cq, const float* ck,
                                   const int32_t* offsets_k, const float* disp, float tau,
                                   uint32_t* sel, cudaStream_t stream);
cudaError_t launch_cluster_stats(int32_t BH, int32_t N, int32_t D, int32_t C, const svg_bf16* v,
                                 const int32_t* order, const int32_t* offsets, float* vbar,
                                 float* disp, cudaStream_t stream);
size_t ear_workspace_bytes(int32_t BH, int32_t D, int32_t C);
cudaError_t launch_ear_compensate(int32_t BH, int32_t N, int32_t D, int32_t C, int32_t bk,
                                  float scale, const svg_bf16* qs, const float* kbar,
                                  const float* vbar, const int32_t* offsets_k,
                                  const int32_t* row_ptr, const int32_t* col_idx, svg_bf16* os,
                                  const float* lse, void* ws, int* status, cudaStream_t stream);
cudaError_t launch_tile_csr(int32_t BH, int32_t N, int32_t Cq, int32_t Ck, int32_t bq, int32_t bk,
                            const int32_t* offsets_q, const int32_t* offsets_k, const uint32_t* sel,
                            int32_t* row_ptr, int32_t* col_idx, int64_t capacity, int32_t* counts,
                            int* status, cudaStream_t stream);
cudaError_t launch_permute_rows(int32_t BH, int32_t N, int32_t D, const svg_bf16* x,
                                const int32_t* order, svg_bf16* y, bool scatter, int* status,
                                cudaStream_t stream);

cudaError_t launch_wait_selftest(long long limit_cycles, int* status, cudaStream_t stream);

}  // namespace svg
