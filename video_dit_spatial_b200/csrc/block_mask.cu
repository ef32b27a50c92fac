// Block-mask construction for Sparse VideoGen's block-sparse attention
// (arXiv 2502.01776 abstract: spatial heads attend within nearby frames,
// temporal heads across frames at nearby in-frame positions; the project
// article "Sparse-VideoGen and the sparsity hiding inside video diffusion
// attention" names block sparse attention as the kernel form).
//
// Block (r, c) is on iff some token pair of the two blocks is allowed. In the
// pattern's own layout a query block's video tokens cover an integer interval
// of groups (frames for spatial/frame-major, positions for
// temporal/position-major), so every CSR row is one run of key blocks plus the
// text key blocks (mask_row in internal.h). Each CTA derives the row offsets
// of its rows from the closed-form counts of all earlier rows (a block-wide
// sum, no inter-CTA communication), then every warp writes its rows' column
// lists with coalesced stores.
#include "internal.h"

namespace svg {
namespace {

constexpr int kRowsPerCta = 256;
constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) block_mask_kernel(MaskGeom m, int32_t nqb,
                                                              int32_t* __restrict__ row_ptr,
                                                              int32_t* __restrict__ col_idx) {
  __shared__ int32_t s_count[kRowsPerCta];
  __shared__ int32_t s_off[kRowsPerCta + 1];
  __shared__ long long s_warp[kThreads / 32];
  const int r0 = blockIdx.x * kRowsPerCta;
  const int tid = threadIdx.x;

  // 1) offset of row r0 = sum of the counts of rows [0, r0)
  long long acc = 0;
  for (int r = tid; r < r0; r += kThreads) acc += mask_row(m, r).count();
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((tid & 31) == 0) s_warp[tid >> 5] = acc;

  // 2) counts of this CTA's rows
  const int r = r0 + tid;
  s_count[tid] = (r < nqb) ? mask_row(m, r).count() : 0;
  __syncthreads();

  // 3) exclusive scan of the counts (one thread; 256 adds)
  if (tid == 0) {
    long long base = 0;
    for (int w = 0; w < kThreads / 32; ++w) base += s_warp[w];
    long long run = base;
    for (int i = 0; i < kRowsPerCta; ++i) {
      s_off[i] = static_cast<int32_t>(run);
      run += s_count[i];
    }
    s_off[kRowsPerCta] = static_cast<int32_t>(run);
  }
  __syncthreads();

  if (r < nqb) row_ptr[r] = s_off[tid];
  if (r == nqb - 1) row_ptr[nqb] = s_off[tid] + s_count[tid];

  // 4) column lists: one warp per row, lanes write consecutive entries
  const int warp = tid >> 5, lane = tid & 31;
  for (int i = warp; i < kRowsPerCta; i += kThreads / 32) {
    const int rr = r0 + i;
    if (rr >= nqb) break;
    const MaskRow row = mask_row(m, rr);
    const int n = s_count[i];
    int32_t* out = col_idx + s_off[i];
    for (int k = lane; k < n; k += 32) out[k] = row.at(k);
  }
}

}  // namespace

MaskGeom make_mask_geom(const Dims& d, int32_t kind) {
  MaskGeom m{};
  m.N = d.N;
  m.Nv = d.Nv;
  m.bq = d.bq;
  m.bk = d.bk;
  m.nkb = d.nkb;
  m.dense = kind == SVG_MASK_DENSE ? 1 : 0;
  if (kind == SVG_MASK_TEMPORAL) {
    m.group = d.T;
    m.ngroups = d.P;
    m.band = d.w;
  } else {
    m.group = d.P;
    m.ngroups = d.T;
    m.band = d.s;
  }
  return m;
}

cudaError_t launch_block_mask(const Dims& d, int32_t kind, int32_t* row_ptr, int32_t* col_idx,
                              cudaStream_t stream) {
  const MaskGeom m = make_mask_geom(d, kind);
  const int grid = (d.nqb + kRowsPerCta - 1) / kRowsPerCta;
  block_mask_kernel<<<grid, kThreads, 0, stream>>>(m, d.nqb, row_ptr, col_idx);
  return cudaGetLastError();
}

}  // namespace svg
