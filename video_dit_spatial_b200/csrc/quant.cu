// e4m3 quantisation of V for the FP8 PV product of the block-sparse attention.
// The project article "Sparse-VideoGen and the sparsity hiding inside video
// diffusion attention" (section "Publication record and the road ahead") lists
// FP8 attention as an open item of the project; the pages fix no scheme. This
// one keeps one scale per (head, channel): v8[b,h,j,c] = e4m3(v[b,h,j,c] *
// (448 / amax_c)) with amax_c = max_j |v[b,h,j,c]| over the head's N rows,
// rounded to nearest even (saturating), and the dequantisation scale
// v_scale[b,h,c] = amax_c / 448, so v ~= v8 * v_scale. A channel that is all
// zeros gets scale 0 and codes 0. Each head is read in its own layout: from v
// when labelled spatial, from the position-major copy vp when labelled temporal.
#include "internal.h"
#include "sm100.cuh"

namespace svg {
namespace {

constexpr int kD = 128;                // channels (bytes of one e4m3 row)
constexpr int kVec = 8;                // channels per thread (one 16-byte bf16 load)
constexpr int kRowThreads = kD / kVec;  // 16 threads per row
constexpr int kThreads = 256;
constexpr int kRowsPerPass = kThreads / kRowThreads;  // 16 rows per block per pass
constexpr float kE4m3Max = 448.0f;

__device__ __forceinline__ const svg_bf16* head_src(const svg_bf16* v, const svg_bf16* vp,
                                                    const int8_t* labels, int bh) {
  const bool temporal = labels != nullptr && labels[bh] == SVG_HEAD_TEMPORAL;
  return temporal ? vp : v;
}

__device__ __forceinline__ void unpack8(const uint4 u, float (&x)[kVec]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// amax[bh*D + c] = max over rows of |v| (as the bit pattern of a non-negative
// float, so an integer max orders it; amax must start at zero).
__global__ void __launch_bounds__(kThreads) amax_kernel(const svg_bf16* __restrict__ v,
                                                        const svg_bf16* __restrict__ vp,
                                                        const int8_t* __restrict__ labels,
                                                        int32_t N, int32_t rows_per_block,
                                                        int* __restrict__ amax) {
  __shared__ float red[kRowsPerPass][kD];
  const int bh = blockIdx.y;
  const svg_bf16* src = head_src(v, vp, labels, bh);
  const int cg = threadIdx.x % kRowThreads;  // channel group: channels 8*cg .. +7
  const int r = threadIdx.x / kRowThreads;
  const int r0 = blockIdx.x * rows_per_block;
  const int r1 = min(N, r0 + rows_per_block);
  float m[kVec];
#pragma unroll
  for (int i = 0; i < kVec; ++i) m[i] = 0.0f;
  for (int row = r0 + r; row < r1; row += kRowsPerPass) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(
        src + (static_cast<size_t>(bh) * N + row) * kD) + cg);
    float x[kVec];
    unpack8(u, x);
#pragma unroll
    for (int i = 0; i < kVec; ++i) m[i] = fmaxf(m[i], fabsf(x[i]));
  }
#pragma unroll
  for (int i = 0; i < kVec; ++i) red[r][cg * kVec + i] = m[i];
  __syncthreads();
  if (threadIdx.x < kD) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < kRowsPerPass; ++i) a = fmaxf(a, red[i][threadIdx.x]);
    atomicMax(amax + static_cast<size_t>(bh) * kD + threadIdx.x, __float_as_int(a));
  }
}

// Codes of every row with the head's amax (read from v_scale, still amax).
__global__ void __launch_bounds__(kThreads) quantize_kernel(const svg_bf16* __restrict__ v,
                                                            const svg_bf16* __restrict__ vp,
                                                            const int8_t* __restrict__ labels,
                                                            int32_t N, int32_t rows_per_block,
                                                            const float* __restrict__ amax,
                                                            uint8_t* __restrict__ v8) {
  const int bh = blockIdx.y;
  const svg_bf16* src = head_src(v, vp, labels, bh);
  const int cg = threadIdx.x % kRowThreads;
  const int r = threadIdx.x / kRowThreads;
  float inv[kVec];
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const float a = amax[static_cast<size_t>(bh) * kD + cg * kVec + i];
    inv[i] = a > 0.0f ? __fdiv_rn(kE4m3Max, a) : 0.0f;
  }
  const int r0 = blockIdx.x * rows_per_block;
  const int r1 = min(N, r0 + rows_per_block);
  for (int row = r0 + r; row < r1; row += kRowsPerPass) {
    const size_t off = (static_cast<size_t>(bh) * N + row) * kD;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(src + off) + cg);
    float x[kVec];
    unpack8(u, x);
    uint2 out;
    out.x = pack_e4m3x4(__fmul_rn(x[0], inv[0]), __fmul_rn(x[1], inv[1]),
                        __fmul_rn(x[2], inv[2]), __fmul_rn(x[3], inv[3]));
    out.y = pack_e4m3x4(__fmul_rn(x[4], inv[4]), __fmul_rn(x[5], inv[5]),
                        __fmul_rn(x[6], inv[6]), __fmul_rn(x[7], inv[7]));
    *reinterpret_cast<uint2*>(v8 + off + cg * kVec) = out;
  }
}

__global__ void scale_kernel(float* __restrict__ v_scale, int32_t n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) v_scale[i] = __fdiv_rn(v_scale[i], kE4m3Max);
}

}  // namespace

cudaError_t launch_quantize_v(const Dims& d, const svg_bf16* v, const svg_bf16* vp,
                              const int8_t* labels, uint8_t* v8, float* v_scale,
                              cudaStream_t stream) {
  if (d.d != kD) return cudaErrorNotSupported;
  const int n = d.BH * kD;
  cudaError_t e = cudaMemsetAsync(v_scale, 0, static_cast<size_t>(n) * sizeof(float), stream);
  if (e != cudaSuccess) return e;
  // about 4 blocks per SM over all heads, each a contiguous run of rows
  const int64_t target_blocks = 4 * 148;
  int64_t per_head = (target_blocks + d.BH - 1) / d.BH;
  if (per_head < 1) per_head = 1;
  int32_t rows = static_cast<int32_t>((d.N + per_head - 1) / per_head);
  rows = (rows + kRowsPerPass - 1) / kRowsPerPass * kRowsPerPass;
  const dim3 grid(static_cast<unsigned>((d.N + rows - 1) / rows), static_cast<unsigned>(d.BH));
  amax_kernel<<<grid, kThreads, 0, stream>>>(v, vp, labels, d.N, rows,
                                             reinterpret_cast<int*>(v_scale));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  quantize_kernel<<<grid, kThreads, 0, stream>>>(v, vp, labels, d.N, rows, v_scale, v8);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  scale_kernel<<<(n + 255) / 256, 256, 0, stream>>>(v_scale, n);
  return cudaGetLastError();
}

}  // namespace svg
