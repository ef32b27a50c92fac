// Layout transformation of Sparse VideoGen ("hardware-efficient tensor layout
// transformation", arXiv 2502.01776 abstract): frame-major <-> position-major
// row permutation of [B, H, N, d] bf16 tensors, restricted to temporal heads.
//
// HBM-bound copy. Each destination row (128 or 256 bytes) is written by a team
// of d/8 threads with 16-byte vector loads and stores, so every warp reads and
// writes whole, aligned row segments. The row map is computed per destination
// row (one integer division), the grid is a multiple of the SM count and
// strides over all rows of all selected heads; up to three tensors share one
// launch.
#include "internal.h"

namespace svg {
namespace {

struct PermuteParams {
  const uint4* in[3];
  uint4* out[3];
  const int8_t* labels;  // nullable
  int32_t n_tensors;
  int32_t T, P, N, Nv;
  int32_t vec_per_row;  // d * 2 / 16 (8 or 16)
  int32_t vec_shift;    // log2(vec_per_row)
  int32_t BH;
  int32_t inverse;  // 0: out[pi(i)] = in[i]; 1: out[i] = in[pi(i)]
};

// Source row of destination row r.
__device__ __forceinline__ int32_t source_row(const PermuteParams& p, int32_t r) {
  if (r >= p.Nv) return r;  // text rows stay in place
  if (!p.inverse) {
    // r is position-major: r = pos*T + f  ->  frame-major f*P + pos
    const int32_t pos = r / p.T;
    const int32_t f = r - pos * p.T;
    return f * p.P + pos;
  }
  // r is frame-major: r = f*P + pos  ->  position-major pos*T + f
  const int32_t f = r / p.P;
  const int32_t pos = r - f * p.P;
  return pos * p.T + f;
}

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads) permute_kernel(const __grid_constant__ PermuteParams p) {
  const int64_t vec_per_head = static_cast<int64_t>(p.N) * p.vec_per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int32_t bh = blockIdx.y; bh < p.BH; bh += gridDim.y) {
    if (p.labels != nullptr && p.labels[bh] != SVG_HEAD_TEMPORAL) continue;
    const int64_t head_off = static_cast<int64_t>(bh) * vec_per_head;
    for (int t = 0; t < p.n_tensors; ++t) {
      const uint4* __restrict__ src = p.in[t] + head_off;
      uint4* __restrict__ dst = p.out[t] + head_off;
      int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
      for (; e + (kUnroll - 1) * stride < vec_per_head; e += kUnroll * stride) {
        uint4 buf[kUnroll];
        int64_t di[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int64_t ee = e + u * stride;
          const int32_t r = static_cast<int32_t>(ee >> p.vec_shift);
          const int32_t c = static_cast<int32_t>(ee) & (p.vec_per_row - 1);
          const int64_t si = static_cast<int64_t>(source_row(p, r)) * p.vec_per_row + c;
          di[u] = ee;
          buf[u] = __ldg(src + si);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) dst[di[u]] = buf[u];
      }
      for (; e < vec_per_head; e += stride) {
        const int32_t r = static_cast<int32_t>(e >> p.vec_shift);
        const int32_t c = static_cast<int32_t>(e) & (p.vec_per_row - 1);
        dst[e] = __ldg(src + static_cast<int64_t>(source_row(p, r)) * p.vec_per_row + c);
      }
    }
  }
}

}  // namespace

cudaError_t launch_permute(const Dims& d, int n_tensors, const svg_bf16* const* in,
                           svg_bf16* const* out, const int8_t* labels, bool inverse,
                           cudaStream_t stream) {
  PermuteParams p{};
  for (int t = 0; t < 3; ++t) {
    p.in[t] = t < n_tensors ? reinterpret_cast<const uint4*>(in[t]) : nullptr;
    p.out[t] = t < n_tensors ? reinterpret_cast<uint4*>(out[t]) : nullptr;
  }
  p.labels = labels;
  p.n_tensors = n_tensors;
  p.T = d.T;
  p.P = d.P;
  p.N = d.N;
  p.Nv = d.Nv;
  p.vec_per_row = d.d * 2 / 16;
  p.vec_shift = p.vec_per_row == 16 ? 4 : 3;
  p.BH = d.BH;
  p.inverse = inverse ? 1 : 0;

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Threads per head: enough 16-byte vectors in flight per SM to cover HBM
  // latency; heads spread over grid.y so unselected heads cost one check.
  const int64_t vec_per_head = static_cast<int64_t>(d.N) * p.vec_per_row;
  int64_t bx = (vec_per_head + kThreads * kUnroll - 1) / (kThreads * kUnroll);
  const int64_t per_head_cap = (static_cast<int64_t>(sms) * 16 + d.BH - 1) / d.BH;
  if (bx > per_head_cap) bx = per_head_cap;
  if (bx < 1) bx = 1;
  const int by = d.BH < 65535 ? d.BH : 65535;
  permute_kernel<<<dim3(static_cast<unsigned>(bx), by), kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace svg
