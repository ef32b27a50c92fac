// Semantic-aware permutation (Sparse VideoGen 2). The project article
// "Sparse-VideoGen and the sparsity hiding inside video diffusion attention",
// section "Three generations of the same idea", describes the second
// generation as semantic-aware sparse attention on an efficient token
// permutation, run by a dynamic attention kernel and a flash (batched) k-means
// kernel; the install section names block-sparse attention with varied block
// sizes. The pages give no formula; the rules implemented here are:
//   k-means     per (b, h), Lloyd iterations on the query (resp. key) vectors:
//               initial centroids are the rows floor(c * N / C); each iteration
//               assigns every row to its nearest centroid (squared Euclidean
//               distance with the centroids rounded to bf16, ties to the
//               smaller index) and replaces each centroid by the mean of its
//               members (an empty cluster keeps its centroid);
//   permutation tokens stably sorted by cluster, so each cluster is one run;
//   selection   query cluster a keeps the fewest key clusters, in descending
//               softmax_b(scale * c_q[a] . c_k[b] + log |b|) weight (ties to
//               the smaller index), whose weights reach top_p;
//   attention   block-granular on the sorted layouts: a (query tile, key tile)
//               pair is computed iff a query cluster present in the query tile
//               keeps a key cluster present in the key tile (the block-sparse
//               attention kernel with one CSR per head).
//
// Kernels:
//   kmeans_prep_kernel     fp32 centroids -> bf16 copy + squared norms
//   kmeans_assign_kernel   tcgen05: S = X C^T for 128 rows x all C centroids
//                          in tensor memory, then a per-row argmin of
//                          |c|^2 - 2 x.c (one softmax-style warpgroup)
//   sort_hist / sort_scan / sort_rank   stable counting sort by cluster
//   kmeans_chunk_sum / kmeans_mean kernels   the members' means: run sums
//                          per chunk of sorted positions, then per cluster
//   select_kernel          the top-p key clusters of each query cluster
//   tile_count / tile_fill kernels      per-head CSR of the tile pairs
//   gather / scatter rows  the permutation of Q, K, V and of the output
// All reductions run in a fixed order: results are deterministic.
#include "internal.h"
#include "sm100.cuh"

namespace svg {
namespace {

// ------------------------------------------------------------ assignment
// warps 0-7 argmin (warpgroup g takes the row tiles j with j % 2 == g, in
// tensor-memory buffer g), warp 8 TMA producer, warp 9 MMA issuer
constexpr int kAsgThreads = 320;
constexpr int kAsgProducer = 8;
constexpr int kAsgMma = 9;
constexpr int kAsgXStages = 4;
constexpr int kMaxC = 256;  // centroids per assignment launch (one MMA N)

struct AsgBarriers {
  uint64_t c_full;
  uint64_t x_full[kAsgXStages], x_empty[kAsgXStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
struct AsgCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kXPanel = 128 * 128;      // 128 rows x 128 B
  static constexpr int kXBytes = kPanels * kXPanel;
  static constexpr int kCPanel = kMaxC * 128;    // up to 256 centroid rows x 128 B
  static constexpr int kCBytes = kPanels * kCPanel;
  static constexpr int kOffC = 0;
  static constexpr int kOffX = kOffC + kCBytes;
  static constexpr int kOffNorm = kOffX + kAsgXStages * kXBytes;
  static constexpr int kOffBar = kOffNorm + kMaxC * 4;
  static constexpr int kBarBytes = (static_cast<int>(sizeof(AsgBarriers)) + 127) / 128 * 128;
  static constexpr int kUsed = kOffBar + kBarBytes + 1024;
  // one CTA per SM: each takes all 512 tensor-memory columns
  static constexpr int kSmem = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  static_assert(kOffX % 1024 == 0 && kXBytes % 1024 == 0, "swizzled tiles 1024-aligned");
};

struct __align__(64) AsgParams {
  CUtensorMap tm_x;   // [BH, N, D] bf16, box (64, 128)
  CUtensorMap tm_c;   // [BH, C, D] bf16, box (64, C)
  const float* norms; // [BH, C]
  int32_t* assign;    // [BH, N]
  int* status;
  int32_t N, C, n_tiles, ctas_per_head;
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

template <int D>
__global__ void __launch_bounds__(kAsgThreads, 1)
    kmeans_assign_kernel(const __grid_constant__ AsgParams p) {
  using Cf = AsgCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sC = smem + Cf::kOffC;
  uint8_t* sX = smem + Cf::kOffX;
  float* sNorm = reinterpret_cast<float*>(smem + Cf::kOffNorm);
  AsgBarriers* bar = reinterpret_cast<AsgBarriers*>(smem + Cf::kOffBar);
  volatile int* abort_flag = &bar->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int bh = blockIdx.y;
  // this CTA's row tiles: [t0, t1)
  const int t0 = static_cast<int>(static_cast<long long>(p.n_tiles) * blockIdx.x / p.ctas_per_head);
  const int t1 =
      static_cast<int>(static_cast<long long>(p.n_tiles) * (blockIdx.x + 1) / p.ctas_per_head);
  const int n = t1 - t0;

  if (warp == 0) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 32) {
    mbar_init(&bar->c_full, 1);
    for (int s = 0; s < kAsgXStages; ++s) {
      mbar_init(&bar->x_full[s], 1);
      mbar_init(&bar->x_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->s_empty[s], 128);
    }
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_mbar_init();
  }
  for (int c = tid; c < p.C; c += kAsgThreads)
    sNorm[c] = p.norms[static_cast<size_t>(bh) * p.C + c];
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == kAsgProducer) {
    if (lane_id() == 0 && n > 0) {
      mbar_arrive_expect_tx(&bar->c_full, static_cast<uint32_t>(p.C * D * 2));
      for (int pn = 0; pn < Cf::kPanels; ++pn)
        tma_load_3d(sC + pn * Cf::kCPanel, &p.tm_c, &bar->c_full, pn * 64, 0, bh);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kAsgXStages;
        if (!mbar_wait(&bar->x_empty[st], ((j / kAsgXStages) & 1) ^ 1, abort_flag, p.status))
          break;
        mbar_arrive_expect_tx(&bar->x_full[st], Cf::kXBytes);
        for (int pn = 0; pn < Cf::kPanels; ++pn)
          tma_load_3d(sX + st * Cf::kXBytes + pn * Cf::kXPanel, &p.tm_x, &bar->x_full[st],
                      pn * 64, (t0 + j) * 128, bh);
        issued = j + 1;
      }
      if (*abort_flag) {
        // let every copy started here land before the CTA retires
        long long tw = clock64();
        while (!mbar_try_wait(&bar->c_full, 0) && clock64() - tw < kWaitLimitCycles) {
        }
        for (int j = (issued > kAsgXStages ? issued - kAsgXStages : 0); j < issued; ++j) {
          tw = clock64();
          while (!mbar_try_wait(&bar->x_full[j % kAsgXStages], (j / kAsgXStages) & 1) &&
                 clock64() - tw < kWaitLimitCycles) {
          }
        }
      }
    }
  } else if (warp == kAsgMma) {
    if (lane_id() == 0 && n > 0) {
      const uint32_t idesc = idesc_bf16_f32(128, p.C, false, false);
      const uint32_t x_addr = smem_u32(sX), c_addr = smem_u32(sC);
      bool ok = mbar_wait(&bar->c_full, 0, abort_flag, p.status);
      for (int j = 0; ok && j < n; ++j) {
        const int xs = j % kAsgXStages, sb = j & 1;
        if (!mbar_wait(&bar->x_full[xs], (j / kAsgXStages) & 1, abort_flag, p.status)) break;
        if (!mbar_wait(&bar->s_empty[sb], ((j >> 1) & 1) ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t s_col = tmem + sb * kMaxC;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          mma_bf16_ss(s_col, sdesc_sw128(x_addr + xs * Cf::kXBytes + (kk >> 2) * Cf::kXPanel + off, 16, 1024),
                      sdesc_sw128(c_addr + (kk >> 2) * Cf::kCPanel + off, 16, 1024), idesc,
                      kk > 0 ? 1u : 0u);
        }
        tc_commit(&bar->s_full[sb]);
        tc_commit(&bar->x_empty[xs]);
      }
      if (*abort_flag) {
        tc_commit(&bar->drain);
        long long tw = clock64();
        while (!mbar_try_wait(&bar->drain, 0) && clock64() - tw < kWaitLimitCycles) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ argmin
    // Four interleaved running minima per row (columns i % 4), each keeping
    // its first minimal column; merged by (distance, column), so the result is
    // the first column of least distance, as a single ascending scan gives.
    const int g = warp >> 2;  // this warpgroup's tensor-memory buffer and tile parity
    const int rl = tid & 127;
    const uint32_t lane_base =
        tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + static_cast<uint32_t>(g * kMaxC);
    for (int j = g; j < n; j += 2) {
      // warp-uniform: the tensor-memory loads below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&bar->s_full[g], (j >> 1) & 1, abort_flag, p.status)))
        break;
      tc_fence_after();
      float best[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
      int best_c[4] = {0, 0, 0, 0};
      for (int ch = 0; ch < p.C / 32; ++ch) {
        uint32_t s[32];
        tmem_ld_32x32b_x32(lane_base + ch * 32, s);
        tmem_ld_wait();
        reg_fence(s);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float dist = fmaf(-2.0f, u2f(s[i]), sNorm[ch * 32 + i]);
          if (dist < best[i & 3]) {  // strict: ties keep the smaller column
            best[i & 3] = dist;
            best_c[i & 3] = ch * 32 + i;
          }
        }
      }
      if (p.C % 32 != 0) {
        // the last 16 columns of a C that is a multiple of 16 but not of 32
        uint32_t s[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(s[0]), "=r"(s[1]), "=r"(s[2]), "=r"(s[3]), "=r"(s[4]), "=r"(s[5]),
              "=r"(s[6]), "=r"(s[7]), "=r"(s[8]), "=r"(s[9]), "=r"(s[10]), "=r"(s[11]),
              "=r"(s[12]), "=r"(s[13]), "=r"(s[14]), "=r"(s[15])
            : "r"(lane_base + (p.C / 32) * 32)
            : "memory");
        tmem_ld_wait();
        reg_fence(s);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = (p.C / 32) * 32 + i;
          const float dist = fmaf(-2.0f, u2f(s[i]), sNorm[c]);
          if (dist < best[i & 3]) {
            best[i & 3] = dist;
            best_c[i & 3] = c;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar->s_empty[g]);
      float b = best[0];
      int bc = best_c[0];
#pragma unroll
      for (int k = 1; k < 4; ++k)
        if (best[k] < b || (best[k] == b && best_c[k] < bc)) {
          b = best[k];
          bc = best_c[k];
        }
      const int row = (t0 + j) * 128 + rl;
      if (row < p.N) p.assign[static_cast<size_t>(bh) * p.N + row] = bc;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// centroids (fp32) -> bf16 copy and squared norms of the bf16 values (fp32,
// channel order). One warp per centroid.
__global__ void kmeans_prep_kernel(const float* __restrict__ cent, int32_t rows, int32_t D,
                                   svg_bf16* __restrict__ cent_bf16, float* __restrict__ norms) {
  const int r = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float acc = 0.0f;
  for (int c0 = 0; c0 < D; c0 += 32) {
    const float x = cent[static_cast<size_t>(r) * D + c0 + lane];
    const uint32_t b = pack_bf16x2(x, 0.0f) & 0xffffu;  // round to nearest even
    cent_bf16[static_cast<size_t>(r) * D + c0 + lane] = static_cast<svg_bf16>(b);
    const float xb = __uint_as_float(b << 16);
    // fixed order: lane partials, then the warp's lanes in order
    acc = fmaf(xb, xb, acc);
  }
  float tot = 0.0f;
  for (int l = 0; l < 32; ++l) tot += __shfl_sync(0xffffffffu, acc, l);
  if (lane == 0) norms[r] = tot;
}

// initial centroids: row floor(c * N / C) of each head
__global__ void kmeans_init_kernel(const svg_bf16* __restrict__ x, int32_t N, int32_t D,
                                   int32_t C, float* __restrict__ cent) {
  const int bh = blockIdx.y, c = blockIdx.x;
  const int64_t row = static_cast<int64_t>(c) * N / C;
  for (int i = threadIdx.x; i < D; i += blockDim.x)
    cent[(static_cast<size_t>(bh) * C + c) * D + i] =
        __uint_as_float(static_cast<uint32_t>(x[(static_cast<size_t>(bh) * N + row) * D + i]) << 16);
}

// ------------------------------------------------------------ stable sort
constexpr int kSortRows = 1024;  // rows per sort block

// hist[bh][blk][c] = rows of block blk in cluster c
__global__ void sort_hist_kernel(const int32_t* __restrict__ assign, int32_t N, int32_t C,
                                 int32_t nblk, int32_t* __restrict__ hist, int* status) {
  extern __shared__ int cnt[];
  const int bh = blockIdx.y, blk = blockIdx.x;
  for (int c = threadIdx.x; c < C; c += blockDim.x) cnt[c] = 0;
  __syncthreads();
  const int r0 = blk * kSortRows, r1 = min(N, r0 + kSortRows);
  for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
    const int a = assign[static_cast<size_t>(bh) * N + r];
    if (a >= 0 && a < C) atomicAdd(&cnt[a], 1);
    else atomicOr(status, kDevErrBounds);
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x)
    hist[(static_cast<size_t>(bh) * nblk + blk) * C + c] = cnt[c];
}

// Per head: offsets[c] = rows in clusters < c; hist becomes each block's first
// sorted position per cluster (offsets[c] + rows of earlier blocks in c).
// Thread c walks cluster c's column of the histogram, kScanBatch blocks of
// loads in flight; the cluster totals are scanned across the CTA (C <= 256 =
// blockDim.x).
constexpr int kScanBatch = 16;

__global__ void __launch_bounds__(256)
    sort_scan_kernel(int32_t* __restrict__ hist, int32_t N, int32_t C, int32_t nblk,
                     int32_t* __restrict__ offsets) {
  __shared__ int warp_tot[8];
  const int bh = blockIdx.x;
  const int c = threadIdx.x, lane = c & 31, wid = c >> 5;
  int32_t* h = hist + static_cast<size_t>(bh) * nblk * C;
  int run = 0;
  if (c < C) {
    for (int b0 = 0; b0 < nblk; b0 += kScanBatch) {
      int v[kScanBatch];
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i)
        v[i] = b0 + i < nblk ? h[static_cast<size_t>(b0 + i) * C + c] : 0;
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i) {
        if (b0 + i < nblk) h[static_cast<size_t>(b0 + i) * C + c] = run;
        run += v[i];
      }
    }
  }
  // exclusive scan of the cluster totals over c
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < wid; ++w) before += warp_tot[w];
  const int first = before + incl - run;  // rows in clusters < c
  if (c < C) offsets[static_cast<size_t>(bh) * (C + 1) + c] = first;
  if (c == C - 1) offsets[static_cast<size_t>(bh) * (C + 1) + C] = first + run;
  if (c < C) {
    for (int b0 = 0; b0 < nblk; b0 += kScanBatch) {
      int v[kScanBatch];
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i)
        v[i] = b0 + i < nblk ? h[static_cast<size_t>(b0 + i) * C + c] : 0;
#pragma unroll
      for (int i = 0; i < kScanBatch; ++i)
        if (b0 + i < nblk) h[static_cast<size_t>(b0 + i) * C + c] = v[i] + first;
    }
  }
}

// One warp per block: walks its rows in order, 32 at a time, and gives each
// the next free sorted position of its cluster (stable).
__global__ void sort_rank_kernel(const int32_t* __restrict__ assign, const int32_t* __restrict__ hist,
                                 int32_t N, int32_t C, int32_t nblk, int32_t* __restrict__ order) {
  extern __shared__ int next[];
  const int bh = blockIdx.y, blk = blockIdx.x;
  const int lane = threadIdx.x;
  for (int c = lane; c < C; c += 32) next[c] = hist[(static_cast<size_t>(bh) * nblk + blk) * C + c];
  __syncwarp();
  const int r0 = blk * kSortRows, r1 = min(N, r0 + kSortRows);
  for (int base = r0; base < r1; base += 32) {
    const int r = base + lane;
    int a = r < r1 ? assign[static_cast<size_t>(bh) * N + r] : -1;
    if (a >= C) a = -1;  // flagged by the histogram
    const unsigned live = __ballot_sync(0xffffffffu, a >= 0);
    const unsigned peers = __match_any_sync(0xffffffffu, a) & live;
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int pos = 0;
    if (a >= 0) pos = next[a] + rank;
    __syncwarp();
    if (a >= 0 && rank == 0) next[a] += __popc(peers);
    __syncwarp();
    if (a >= 0) order[static_cast<size_t>(bh) * N + pos] = r;
  }
}

// ------------------------------------------------------------ cluster sums
// Members of a cluster, summed by one CTA of kSumWarps warps (the value
// statistics of SVG-EAR): warp w takes the
// w-th of kSumWarps equal runs of the cluster's sorted positions and adds its
// rows in order (kBatch row loads in flight), lane l holding channels
// [D/32 * l, D/32 * (l+1)); the warps' partial sums are then added in warp
// order. The order of every addition is fixed: the result is deterministic.
constexpr int kSumWarps = 4;
constexpr int kBatch = 8;

template <int D>
__device__ __forceinline__ void load_row_slice(const svg_bf16* __restrict__ x, size_t row,
                                               int lane, float (&out)[D / 32]) {
  const svg_bf16* src = x + row * D + lane * (D / 32);
  if constexpr (D / 32 == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    out[0] = __uint_as_float(u.x << 16);
    out[1] = __uint_as_float(u.x & 0xffff0000u);
    out[2] = __uint_as_float(u.y << 16);
    out[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(src);
    out[0] = __uint_as_float(u << 16);
    out[1] = __uint_as_float(u & 0xffff0000u);
  }
}

// sum[i] += the rows at sorted positions [q0, q1) of head bh, in order (or,
// with center, their squared deviations from it)
template <int D>
__device__ __forceinline__ void sum_rows(const svg_bf16* __restrict__ x,
                                         const int32_t* __restrict__ order, int32_t N, int bh,
                                         int q0, int q1, int lane, float (&sum)[D / 32],
                                         const float* center) {
  constexpr int kPer = D / 32;
  const int32_t* ord = order + static_cast<size_t>(bh) * N;
  for (int base = q0; base < q1; base += kBatch) {
    float v[kBatch][kPer];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (base + u < q1)
        load_row_slice<D>(x, static_cast<size_t>(bh) * N + __ldg(ord + base + u), lane, v[u]);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (base + u >= q1) break;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        if (center == nullptr) {
          sum[i] += v[u][i];
        } else {
          const float dv = v[u][i] - center[i];
          sum[i] = fmaf(dv, dv, sum[i]);
        }
      }
    }
  }
}

// ------------------------------------------------------------ update
// Two passes in a fixed summation order, with work per warp bounded by a
// chunk whatever the cluster sizes. The sorted positions of a head are cut
// into chunks of kChunkRows. Warp i of the first pass adds, in order, the rows
// of each cluster's run inside chunk i, and stores each run's sum as the
// partial of (chunk i, cluster c). When chunk i meets cluster c and chunk i'
// meets cluster c' != c with i + c = i' + c', one cluster would have to end
// past the start of the other, so slot i + c (fewer than nchunks + C slots per
// head) is unique. The second pass adds each cluster's partials in chunk order
// and divides by the member count.
constexpr int kChunkRows = 256;
constexpr int kChunkWarps = 4;
constexpr int kChunkBatch = 16;   // rows per pipeline stage
constexpr int kChunkStages = 4;   // stages per warp (kChunkStages - 1 batches in flight)

template <int D>
struct ChunkCfg {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kLanesPerRow = kRowBytes / 16;  // 16-byte copies per row
  static constexpr int kRowsPerCopy = 32 / kLanesPerRow;
  static constexpr int kStageBytes = kChunkBatch * kRowBytes;
  static constexpr int kWarpBytes = kChunkStages * kStageBytes + kChunkRows * 4;
  static constexpr int kSmem = kChunkWarps * kWarpBytes;
  static_assert(kChunkBatch % kRowsPerCopy == 0, "a stage is whole copy instructions");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One warp per chunk. The chunk's rows stream through a ring of kChunkStages
// shared-memory stages of kChunkBatch rows (cp.async, 16 bytes per lane), so
// the next batches are in flight while one is added; lane l adds channels
// [D/32 * l, D/32 * (l+1)) of each row in sorted order.
template <int D>
__global__ void __launch_bounds__(32 * kChunkWarps)
    kmeans_chunk_sum_kernel(const svg_bf16* __restrict__ x, const int32_t* __restrict__ order,
                            const int32_t* __restrict__ offsets, int32_t N, int32_t C,
                            int32_t nchunks, float* __restrict__ partial, int* status) {
  using Cf = ChunkCfg<D>;
  constexpr int kPer = D / 32;
  extern __shared__ __align__(16) uint8_t chunk_smem[];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kChunkWarps + w;
  const int bh = blockIdx.y;
  if (chunk >= nchunks) return;
  uint8_t* ring = chunk_smem + w * Cf::kWarpBytes;
  int32_t* rows_s = reinterpret_cast<int32_t*>(ring + kChunkStages * Cf::kStageBytes);
  const int p0 = chunk * kChunkRows, p1 = min(N, p0 + kChunkRows);
  const int32_t* off = offsets + static_cast<size_t>(bh) * (C + 1);
  const int32_t* ord = order + static_cast<size_t>(bh) * N;
  for (int q = lane; q < p1 - p0; q += 32) {
    int r = __ldg(ord + p0 + q);
    if (r < 0 || r >= N) {  // only if an earlier step failed: flag it, read row 0
      atomicOr(status, kDevErrBounds);
      r = 0;
    }
    rows_s[q] = r;
  }
  __syncwarp();
  const svg_bf16* xh = x + static_cast<size_t>(bh) * N * D;
  const int nb = (p1 - p0 + kChunkBatch - 1) / kChunkBatch;
  const int sub = lane % Cf::kLanesPerRow, row_in_copy = lane / Cf::kLanesPerRow;
  auto issue = [&](int bt) {
    if (bt < nb) {
      const uint32_t st = smem_u32(ring + (bt % kChunkStages) * Cf::kStageBytes);
#pragma unroll
      for (int i = 0; i < kChunkBatch / Cf::kRowsPerCopy; ++i) {
        const int u = i * Cf::kRowsPerCopy + row_in_copy;
        const int q = bt * kChunkBatch + u;
        if (p0 + q < p1)
          cp_async16(st + u * Cf::kRowBytes + sub * 16,
                     xh + static_cast<size_t>(rows_s[q]) * D + sub * 8);
      }
    }
    cp_async_commit();  // an empty group past the end keeps the wait count uniform
  };
#pragma unroll
  for (int s = 0; s < kChunkStages - 1; ++s) issue(s);
  // the cluster of position p0: the last c with off[c] <= p0 (it is not empty)
  int n_le = 0;
  for (int k = lane; k <= C; k += 32) n_le += __ldg(off + k) <= p0 ? 1 : 0;
#pragma unroll
  for (int o = 16; o; o >>= 1) n_le += __shfl_xor_sync(0xffffffffu, n_le, o);
  // (C - 1 at most: the positions of rows an earlier failed step left unsorted
  // lie past off[C])
  int c = min(n_le - 1, C - 1);
  int next = __ldg(off + c + 1);
  float* part = partial + static_cast<size_t>(bh) * (nchunks + C) * D + lane * kPer;
  float sum[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) sum[i] = 0.0f;
  for (int bt = 0; bt < nb; ++bt) {
    issue(bt + kChunkStages - 1);  // into the stage added in the previous iteration
    cp_async_wait<kChunkStages - 1>();
    __syncwarp();
    const uint8_t* st = ring + (bt % kChunkStages) * Cf::kStageBytes + lane * kPer * 2;
#pragma unroll 4
    for (int u = 0; u < kChunkBatch; ++u) {
      const int p = p0 + bt * kChunkBatch + u;
      if (p >= p1) break;
      float v[kPer];
      if constexpr (kPer == 4) {
        const uint2 r = *reinterpret_cast<const uint2*>(st + u * Cf::kRowBytes);
        v[0] = __uint_as_float(r.x << 16);
        v[1] = __uint_as_float(r.x & 0xffff0000u);
        v[2] = __uint_as_float(r.y << 16);
        v[3] = __uint_as_float(r.y & 0xffff0000u);
      } else {
        const uint32_t r = *reinterpret_cast<const uint32_t*>(st + u * Cf::kRowBytes);
        v[0] = __uint_as_float(r << 16);
        v[1] = __uint_as_float(r & 0xffff0000u);
      }
      if (p >= next) {  // cluster c ends before p: store its run, find p's cluster
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
          part[static_cast<size_t>(chunk + c) * D + i] = sum[i];
          sum[i] = 0.0f;
        }
        while (p >= next && c < C - 1) next = __ldg(off + (++c) + 1);
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) sum[i] += v[i];
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  cp_async_wait<0>();
#pragma unroll
  for (int i = 0; i < kPer; ++i) part[static_cast<size_t>(chunk + c) * D + i] = sum[i];
}

template <int D>
__global__ void __launch_bounds__(32 * kChunkWarps)
    kmeans_mean_kernel(const float* __restrict__ partial, const int32_t* __restrict__ offsets,
                       int32_t C, int32_t nchunks, const float* __restrict__ c_in,
                       float* __restrict__ c_out) {
  constexpr int kPer = D / 32;
  constexpr int kInFlight = 8;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x * kChunkWarps + (threadIdx.x >> 5);
  const int bh = blockIdx.y;
  if (c >= C) return;
  const int32_t* off = offsets + static_cast<size_t>(bh) * (C + 1);
  const int p0 = __ldg(off + c), p1 = __ldg(off + c + 1);
  float* dst = c_out + (static_cast<size_t>(bh) * C + c) * D + lane * kPer;
  if (p1 <= p0) {
    const float* prev = c_in + (static_cast<size_t>(bh) * C + c) * D + lane * kPer;
#pragma unroll
    for (int i = 0; i < kPer; ++i) dst[i] = prev[i];
    return;
  }
  const int i0 = p0 / kChunkRows, i1 = (p1 - 1) / kChunkRows;
  const float* part = partial + static_cast<size_t>(bh) * (nchunks + C) * D + lane * kPer;
  float tot[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) tot[i] = 0.0f;
  for (int ib = i0; ib <= i1; ib += kInFlight) {
    float v[kInFlight][kPer];
#pragma unroll
    for (int u = 0; u < kInFlight; ++u)
      if (ib + u <= i1) {
        const float* src = part + static_cast<size_t>(ib + u + c) * D;
#pragma unroll
        for (int i = 0; i < kPer; ++i) v[u][i] = src[i];
      }
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      if (ib + u > i1) break;
#pragma unroll
      for (int i = 0; i < kPer; ++i) tot[i] += v[u][i];
    }
  }
  const float n = static_cast<float>(p1 - p0);
#pragma unroll
  for (int i = 0; i < kPer; ++i) dst[i] = __fdiv_rn(tot[i], n);
}

// ------------------------------------------------------------ selection
// One CTA per (bh, group of kSelGroup query clusters); the group's centroids
// are staged in shared memory. Each warp forms the kSelGroup dot products of
// its share of the key clusters, lane l taking channels l, l + 32, ... (the
// key centroid is read once per group, coalesced) and the lanes' partial sums
// added by a butterfly. Thread b then handles key cluster b: for each query
// cluster of the group the weights, their maximum and their sum are formed as
// for a lone cluster.
// With disp != nullptr (SVG-EAR), a skipped cluster is kept anyway when its
// error estimate w_b * disp_b exceeds tau.
constexpr int kSelGroup = 8;

__global__ void select_kernel(const float* __restrict__ cq, const float* __restrict__ ck,
                              const int32_t* __restrict__ offsets_k, int32_t D, int32_t Cq,
                              int32_t Ck, float scale, float top_p, const float* __restrict__ disp,
                              float tau, uint32_t* __restrict__ sel) {
  // [kSelGroup][Ck] weights (first the dot products), [kSelGroup][32]
  // reduction slots, then [kSelGroup][D] query centroids
  extern __shared__ float w[];
  float* red = w + kSelGroup * Ck;
  float* xs = red + kSelGroup * 32;
  const int a0 = blockIdx.x * kSelGroup, bh = blockIdx.y;
  const int na = min(kSelGroup, Cq - a0);
  const int b = threadIdx.x;
  const int lane = b & 31, wid = b >> 5, nw = blockDim.x >> 5;
  const int words = (Ck + 31) / 32;
  const int32_t* off = offsets_k + static_cast<size_t>(bh) * (Ck + 1);
  {
    const float* x = cq + (static_cast<size_t>(bh) * Cq + a0) * D;
    for (int i = b; i < kSelGroup * D; i += blockDim.x) xs[i] = i < na * D ? x[i] : 0.0f;
  }
  __syncthreads();
  for (int kb = wid; kb < Ck; kb += nw) {
    if (off[kb + 1] - off[kb] <= 0) continue;  // warp-uniform
    const float* y = ck + (static_cast<size_t>(bh) * Ck + kb) * D;
    float acc[kSelGroup];
#pragma unroll
    for (int g = 0; g < kSelGroup; ++g) acc[g] = 0.0f;
    for (int i = lane; i < D; i += 32) {
      const float yi = y[i];
#pragma unroll
      for (int g = 0; g < kSelGroup; ++g) acc[g] = fmaf(xs[g * D + i], yi, acc[g]);
    }
#pragma unroll
    for (int g = 0; g < kSelGroup; ++g) {
      for (int o = 16; o > 0; o >>= 1) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < kSelGroup; ++g) w[g * Ck + kb] = acc[g];
    }
  }
  __syncthreads();
  float z[kSelGroup];
#pragma unroll
  for (int g = 0; g < kSelGroup; ++g) z[g] = -INFINITY;
  int size = 0;
  if (b < Ck) {
    size = off[b + 1] - off[b];
    if (size > 0) {
      const float ls = logf(static_cast<float>(size));
#pragma unroll
      for (int g = 0; g < kSelGroup; ++g) z[g] = fmaf(scale, w[g * Ck + b], ls);
    }
  }
  __syncthreads();  // the dot products are read; w now takes the weights
  // block maxima
  float m[kSelGroup];
#pragma unroll
  for (int g = 0; g < kSelGroup; ++g) {
    m[g] = z[g];
    for (int o = 16; o > 0; o >>= 1) m[g] = fmaxf(m[g], __shfl_xor_sync(0xffffffffu, m[g], o));
    if (lane == 0) red[g * 32 + wid] = m[g];
  }
  __syncthreads();
#pragma unroll
  for (int g = 0; g < kSelGroup; ++g) {
    m[g] = -INFINITY;
    for (int i = 0; i < nw; ++i) m[g] = fmaxf(m[g], red[g * 32 + i]);
  }
  __syncthreads();
  // block sums in a fixed order
  float e[kSelGroup];
#pragma unroll
  for (int g = 0; g < kSelGroup; ++g) {
    e[g] = (b < Ck && size > 0) ? expf(z[g] - m[g]) : 0.0f;
    float s = e[g];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[g * 32 + wid] = s;
  }
  __syncthreads();
  float wb[kSelGroup];
#pragma unroll
  for (int g = 0; g < kSelGroup; ++g) {
    float tot = 0.0f;
    for (int i = 0; i < nw; ++i) tot += red[g * 32 + i];
    wb[g] = e[g] / tot;
    if (b < Ck) w[g * Ck + b] = wb[g];
  }
  __syncthreads();
  const float db = (disp != nullptr && b < Ck) ? disp[static_cast<size_t>(bh) * Ck + b] : 0.0f;
#pragma unroll
  for (int g = 0; g < kSelGroup; ++g) {
    if (g >= na) break;
    bool keep = false;
    if (b < Ck && size > 0) {
      // weight of the clusters ranked before b (descending weight, ties by index)
      const float* wg = w + g * Ck;
      float before = 0.0f;
      for (int i = 0; i < Ck; ++i) {
        const float wi = wg[i];
        if (wi > wb[g] || (wi == wb[g] && i < b)) before += wi;
      }
      keep = before < top_p;
      if (!keep && disp != nullptr) keep = wb[g] * db > tau;
    }
    const unsigned bits = __ballot_sync(0xffffffffu, keep);
    if (lane == 0 && wid < words) sel[(static_cast<size_t>(bh) * Cq + a0 + g) * words + wid] = bits;
  }
}

// ------------------------------------------------------------ tile CSR
constexpr int kTileWarps = 4;
constexpr int kMaxSelWords = 32;    // Ck <= 1024
constexpr int kMaxTileWords = 128;  // key tiles <= 4096

// The key tiles of query tile r of head bh, as a bitmap in `tiles` (the
// warp's shared words). Query clusters present in the tile: the clusters of
// its first and last sorted positions and all between them.
__device__ void tile_key_bitmap(const int32_t* __restrict__ offq, const int32_t* __restrict__ offk,
                                const uint32_t* __restrict__ sel_bh, int32_t N, int32_t Cq,
                                int32_t Ck, int32_t bq, int32_t bk, int32_t nkb, int r,
                                uint32_t* keep, uint32_t* tiles) {
  const int lane = threadIdx.x & 31;
  const int sw = (Ck + 31) / 32, tw = (nkb + 31) / 32;
  const int p0 = r * bq, p1 = min(N, p0 + bq) - 1;
  // cluster of a sorted position: the last a with offq[a] <= pos
  auto cluster_at = [&](int pos) {
    int lo = 0, hi = Cq - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (offq[mid] <= pos) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  const int a0 = cluster_at(p0), a1 = cluster_at(p1);
  for (int i = lane; i < sw; i += 32) {
    uint32_t m = 0;
    for (int a = a0; a <= a1; ++a)  // clusters with no position in the tile do not count
      if (offq[a + 1] > offq[a]) m |= sel_bh[static_cast<size_t>(a) * sw + i];
    keep[i] = m;
  }
  for (int i = lane; i < tw; i += 32) tiles[i] = 0;
  __syncwarp();
  for (int b = lane; b < Ck; b += 32) {
    if (!((keep[b >> 5] >> (b & 31)) & 1u)) continue;
    const int k0 = offk[b], k1 = offk[b + 1];
    if (k1 <= k0) continue;
    for (int t = k0 / bk; t <= (k1 - 1) / bk; ++t) atomicOr(&tiles[t >> 5], 1u << (t & 31));
  }
  __syncwarp();
}

__global__ void tile_count_kernel(const int32_t* __restrict__ offsets_q,
                                  const int32_t* __restrict__ offsets_k,
                                  const uint32_t* __restrict__ sel, int32_t BH, int32_t N,
                                  int32_t Cq, int32_t Ck, int32_t bq, int32_t bk, int32_t nqb,
                                  int32_t nkb, int32_t* __restrict__ counts) {
  __shared__ uint32_t keep[kTileWarps][kMaxSelWords];
  __shared__ uint32_t tiles[kTileWarps][kMaxTileWords];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kTileWarps + w;
  if (row >= BH * nqb) return;
  const int bh = row / nqb, r = row - bh * nqb;
  const int sw = (Ck + 31) / 32, tw = (nkb + 31) / 32;
  tile_key_bitmap(offsets_q + static_cast<size_t>(bh) * (Cq + 1),
                  offsets_k + static_cast<size_t>(bh) * (Ck + 1),
                  sel + static_cast<size_t>(bh) * Cq * sw, N, Cq, Ck, bq, bk, nkb, r, keep[w],
                  tiles[w]);
  int c = 0;
  for (int i = lane; i < tw; i += 32) c += __popc(tiles[w][i]);
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) counts[row] = c;
}

// row_ptr[0] = 0, row_ptr[i+1] = row_ptr[i] + counts[i] (one CTA, fixed order)
__global__ void tile_scan_kernel(const int32_t* __restrict__ counts, int32_t rows,
                                 int32_t* __restrict__ row_ptr) {
  __shared__ int32_t part[1024];
  const int t = threadIdx.x, nt = blockDim.x;
  const int per = (rows + nt - 1) / nt;
  const int i0 = t * per, i1 = min(rows, i0 + per);
  int32_t s = 0;
  for (int i = i0; i < i1; ++i) s += counts[i];
  part[t] = s;
  __syncthreads();
  if (t == 0) {
    int32_t run = 0;
    for (int i = 0; i < nt; ++i) {
      const int32_t v = part[i];
      part[i] = run;
      run += v;
    }
    row_ptr[rows] = run;
  }
  __syncthreads();
  int32_t run = part[t];
  for (int i = i0; i < i1; ++i) {
    row_ptr[i] = run;
    run += counts[i];
  }
}

__global__ void tile_fill_kernel(const int32_t* __restrict__ offsets_q,
                                 const int32_t* __restrict__ offsets_k,
                                 const uint32_t* __restrict__ sel, int32_t BH, int32_t N, int32_t Cq,
                                 int32_t Ck, int32_t bq, int32_t bk, int32_t nqb, int32_t nkb,
                                 const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
                                 int64_t capacity, int* status) {
  __shared__ uint32_t keep[kTileWarps][kMaxSelWords];
  __shared__ uint32_t tiles[kTileWarps][kMaxTileWords];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kTileWarps + w;
  if (row >= BH * nqb) return;
  const int bh = row / nqb, r = row - bh * nqb;
  const int sw = (Ck + 31) / 32, tw = (nkb + 31) / 32;
  tile_key_bitmap(offsets_q + static_cast<size_t>(bh) * (Cq + 1),
                  offsets_k + static_cast<size_t>(bh) * (Ck + 1),
                  sel + static_cast<size_t>(bh) * Cq * sw, N, Cq, Ck, bq, bk, nkb, r, keep[w],
                  tiles[w]);
  int64_t pos = row_ptr[row];
  for (int i0 = 0; i0 < tw; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t bits = i < tw ? tiles[w][i] : 0u;
    const int c = __popc(bits);
    int incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int64_t p = pos + incl - c;
    for (uint32_t m = bits; m; m &= m - 1) {
      const int t = 32 * i + __ffs(m) - 1;
      if (p < capacity) col_idx[p] = t;
      else atomicOr(status, kDevErrBounds);
      ++p;
    }
    pos += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// ------------------------------------------------------------ row permutation
// gather: y[bh, pos] = x[bh, order[bh, pos]];  scatter: y[bh, order[bh, pos]] = x[bh, pos]
template <bool kScatter>
__global__ void permute_rows_kernel(const svg_bf16* __restrict__ x, const int32_t* __restrict__ order,
                                    int32_t BH, int32_t N, int32_t D, svg_bf16* __restrict__ y,
                                    int* status) {
  const int vec = D / 8;  // 16-byte vectors per row
  const int64_t total = static_cast<int64_t>(BH) * N * vec;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t rowi = i / vec;  // bh * N + sorted position
    const int v = static_cast<int>(i - rowi * vec);
    const int64_t bh = rowi / N;
    const int r = order[rowi];
    if (r < 0 || r >= N) {
      atomicOr(status, kDevErrBounds);
      continue;
    }
    const int64_t src = kScatter ? rowi : bh * N + r;
    const int64_t dst = kScatter ? bh * N + r : rowi;
    reinterpret_cast<uint4*>(y + dst * D)[v] = reinterpret_cast<const uint4*>(x + src * D)[v];
  }
}

// ------------------------------------------------------------ SVG-EAR
// Per key cluster (one CTA of kSumWarps warps per (bh, b), the update kernel's
// fixed split and order), over its members in sorted order: vbar = the fp32
// mean value, disp = sqrt(mean over members and channels of (v - vbar)^2); an
// empty cluster gets zeros.
template <int D>
__global__ void __launch_bounds__(32 * kSumWarps)
    cluster_stats_kernel(const svg_bf16* __restrict__ v, const int32_t* __restrict__ order,
                         const int32_t* __restrict__ offsets, int32_t N, int32_t C,
                         float* __restrict__ vbar, float* __restrict__ disp) {
  constexpr int kPer = D / 32;
  __shared__ float part[kSumWarps][D];
  __shared__ float mean_s[D];
  __shared__ float sq_s[kSumWarps];
  const int c = blockIdx.x, bh = blockIdx.y;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* off = offsets + static_cast<size_t>(bh) * (C + 1);
  const int p0 = off[c], p1 = off[c + 1], cnt = p1 - p0;
  const int q0 = p0 + static_cast<int>(static_cast<long long>(cnt) * w / kSumWarps);
  const int q1 = p0 + static_cast<int>(static_cast<long long>(cnt) * (w + 1) / kSumWarps);
  float acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.0f;
  sum_rows<D>(v, order, N, bh, q0, q1, lane, acc, nullptr);
#pragma unroll
  for (int i = 0; i < kPer; ++i) part[w][lane * kPer + i] = acc[i];
  __syncthreads();
  if (w == 0) {
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      float tot = 0.0f;
#pragma unroll
      for (int ww = 0; ww < kSumWarps; ++ww) tot += part[ww][lane * kPer + i];
      mean_s[lane * kPer + i] = cnt > 0 ? __fdiv_rn(tot, static_cast<float>(cnt)) : 0.0f;
    }
  }
  __syncthreads();
  float center[kPer], sq[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    center[i] = mean_s[lane * kPer + i];
    sq[i] = 0.0f;
  }
  sum_rows<D>(v, order, N, bh, q0, q1, lane, sq, center);
  float lane_sq = 0.0f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) lane_sq += sq[i];
  float wsum = 0.0f;
  for (int l = 0; l < 32; ++l) wsum += __shfl_sync(0xffffffffu, lane_sq, l);
  if (lane == 0) sq_s[w] = wsum;
  __syncthreads();
  if (w == 0) {
    float* dst = vbar + (static_cast<size_t>(bh) * C + c) * D + lane * kPer;
#pragma unroll
    for (int i = 0; i < kPer; ++i) dst[i] = mean_s[lane * kPer + i];
    if (lane == 0) {
      float tot = 0.0f;
      for (int ww = 0; ww < kSumWarps; ++ww) tot += sq_s[ww];
      disp[static_cast<size_t>(bh) * C + c] =
          cnt > 0 ? sqrtf(__fdiv_rn(tot, static_cast<float>(cnt) * D)) : 0.0f;
    }
  }
}

// fp32 [rows, D] -> bf16 [rows, D] (round to nearest even)
__global__ void to_bf16_kernel(const float* __restrict__ x, int64_t n, svg_bf16* __restrict__ y) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = static_cast<svg_bf16>(pack_bf16x2(x[i], 0.0f) & 0xffffu);
}

// Centroid compensation of sorted query tiles (128 rows) of head bh:
//   bias_b = log2(n_b), n_b = keys of cluster b outside the tile's computed key
//            tiles (-inf when none);
//   S = Q kbar^T (tcgen05, 128 x Ck), z_b = S_b * scale * log2(e) + bias_b,
//   P = 2^(z - max z) (bf16, in tensor memory), O_c = P vbar (tcgen05);
// then merged with the block-sparse output of the same rows through its
// log-sum-exp: O = (O_s e^lse + O_c 2^m) / (e^lse + sum P 2^m), in place.
// Persistent: CTA i takes the consecutive tiles [T0, T1) of the (bh, tile)
// order, loads a head's bf16 centroids and value means once, and streams the
// query tiles through two shared-memory buffers. Per tile each of s_full,
// p_full, o_full and o_empty completes once (kv_free once per change of head,
// c_full once per load), and every wait is on a phase that the waiter's own
// earlier step must precede, so no barrier runs two phases ahead of a waiter.
constexpr int kEarThreads = 192;  // warps 0-3 softmax / merge, 4 producer, 5 MMA
constexpr int kEarMaxTiles = 4096;

struct EarBarriers {
  uint64_t c_full, kv_free, q_full[2], q_empty[2], s_full, p_full, o_full, o_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
  uint32_t tiles[kEarMaxTiles / 32];
};

template <int D>
struct EarCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kCPanel = kMaxC * 128;  // up to 256 centroid rows x 128 B
  static constexpr int kCBytes = kPanels * kCPanel;
  static constexpr int kQPanel = 128 * 128;
  static constexpr int kQBytes = kPanels * kQPanel;
  static constexpr int kOffK = 0;               // kbar (K-major operand of S)
  static constexpr int kOffV = kOffK + kCBytes;  // vbar (MN-major operand of O)
  static constexpr int kOffQ = kOffV + kCBytes;  // two query tiles
  static constexpr int kOffBias = kOffQ + 2 * kQBytes;  // two tiles' biases
  static constexpr int kOffBar = kOffBias + 2 * kMaxC * 4;
  static constexpr int kBarBytes = (static_cast<int>(sizeof(EarBarriers)) + 127) / 128 * 128;
  static constexpr int kUsed = kOffBar + kBarBytes + 1024;
  static constexpr int kSmem = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
  static constexpr uint32_t kColS = 0, kColO = 256;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
};

struct __align__(64) EarParams {
  CUtensorMap tm_q;   // sorted queries [BH, N, D], box (64, 128)
  CUtensorMap tm_kb;  // kbar bf16 [BH, C, D], box (64, C)
  CUtensorMap tm_vb;  // vbar bf16 [BH, C, D], box (64, C)
  const int32_t* offsets_k;  // [BH, C+1]
  const int32_t* row_ptr;    // [BH*nqb+1]
  const int32_t* col_idx;
  svg_bf16* os;              // [BH, N, D] sorted sparse output, overwritten
  const float* lse;          // [BH, N] natural log
  int* status;
  int32_t BH, N, C, bk, nqb, nkb;
  float scale_log2;
};

// 16 columns of 32-bit tensor memory of this warp's 32 lanes
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Barrier `id` over `count` threads that also returns the OR of `pred` over them.
__device__ __forceinline__ bool named_bar_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("barrier.cta.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kEarThreads, 1) ear_compensate_kernel(const __grid_constant__ EarParams p) {
  using Cf = EarCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem + Cf::kOffK;
  uint8_t* sV = smem + Cf::kOffV;
  uint8_t* sQ = smem + Cf::kOffQ;
  float* sBias = reinterpret_cast<float*>(smem + Cf::kOffBias);
  EarBarriers* bar = reinterpret_cast<EarBarriers*>(smem + Cf::kOffBar);
  volatile int* abort_flag = &bar->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5;
  // this CTA's tiles: [T0, T0 + n) of the order u = bh * nqb + r
  const long long total = static_cast<long long>(p.BH) * p.nqb;
  const int T0 = static_cast<int>(total * blockIdx.x / gridDim.x);
  const int n = static_cast<int>(total * (blockIdx.x + 1) / gridDim.x) - T0;

  if (warp == 0) {
    tmem_alloc(&bar->tmem_base, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 32) {
    mbar_init(&bar->c_full, 1);
    mbar_init(&bar->kv_free, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar->q_full[b], 1);
      mbar_init(&bar->q_empty[b], 1);
    }
    mbar_init(&bar->s_full, 1);
    mbar_init(&bar->p_full, 128);
    mbar_init(&bar->o_full, 1);
    mbar_init(&bar->o_empty, 128);
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane_id() == 0) {
      int cur = -1, loads = 0, q_issued = 0;
      bool ok = true;
      for (int it = 0; it < n; ++it) {
        const int u = T0 + it, bh = u / p.nqb, r = u - bh * p.nqb;
        if (bh != cur) {
          // the previous head's last product has read its centroids
          if (loads > 0 && !mbar_wait(&bar->kv_free, (loads - 1) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar->c_full, static_cast<uint32_t>(2 * p.C * D * 2));
          for (int pn = 0; pn < Cf::kPanels; ++pn) {
            tma_load_3d(sK + pn * Cf::kCPanel, &p.tm_kb, &bar->c_full, pn * 64, 0, bh);
            tma_load_3d(sV + pn * Cf::kCPanel, &p.tm_vb, &bar->c_full, pn * 64, 0, bh);
          }
          ++loads;
          cur = bh;
        }
        const int b = it & 1;
        if (!mbar_wait(&bar->q_empty[b], ((it >> 1) & 1) ^ 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bar->q_full[b], Cf::kQBytes);
        for (int pn = 0; pn < Cf::kPanels; ++pn)
          tma_load_3d(sQ + b * Cf::kQBytes + pn * Cf::kQPanel, &p.tm_q, &bar->q_full[b],
                      pn * 64, r * 128, bh);
        q_issued = it + 1;
      }
      if (!ok || *abort_flag) {
        // let every copy started here land before the CTA retires (bounded)
        long long tw0 = clock64();
        while (loads > 0 && !mbar_try_wait(&bar->c_full, (loads - 1) & 1) &&
               clock64() - tw0 < kWaitLimitCycles) {
        }
        for (int it = (q_issued > 2 ? q_issued - 2 : 0); it < q_issued; ++it) {
          tw0 = clock64();
          while (!mbar_try_wait(&bar->q_full[it & 1], (it >> 1) & 1) &&
                 clock64() - tw0 < kWaitLimitCycles) {
          }
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane_id() == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, p.C, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      int cur = -1, loads = 0;
      bool ok = true;
      for (int it = 0; it < n && ok; ++it) {
        const int u = T0 + it, bh = u / p.nqb;
        const int b = it & 1;
        if (bh != cur) {
          ok = mbar_wait(&bar->c_full, loads & 1, abort_flag, p.status);
          ++loads;
          cur = bh;
          if (!ok) break;
        }
        if (!mbar_wait(&bar->q_full[b], (it >> 1) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        // S(it) follows O(it-1) in the pipe, which has read P(it-1) from the same columns
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = (kk & 3) * 32;
          mma_bf16_ss(tmem + Cf::kColS,
                      sdesc_sw128(q_addr + b * Cf::kQBytes + (kk >> 2) * Cf::kQPanel + o, 16, 1024),
                      sdesc_sw128(k_addr + (kk >> 2) * Cf::kCPanel + o, 16, 1024), idesc_s,
                      kk > 0 ? 1u : 0u);
        }
        tc_commit(&bar->s_full);
        tc_commit(&bar->q_empty[b]);
        if (!mbar_wait(&bar->p_full, it & 1, abort_flag, p.status)) break;
        // the merge of tile it-1 has read O
        if (it > 0 && !mbar_wait(&bar->o_empty, (it - 1) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        for (int kk = 0; kk < p.C / 16; ++kk)
          mma_bf16_ts(tmem + Cf::kColO, tmem + Cf::kColS + kk * 8,
                      sdesc_sw128(v_addr + kk * 16 * 128, Cf::kCPanel, 1024), idesc_o,
                      kk > 0 ? 1u : 0u);
        tc_commit(&bar->o_full);
        if (it + 1 < n && (u + 1) / p.nqb != bh) tc_commit(&bar->kv_free);
      }
      if (*abort_flag) {
        tc_commit(&bar->drain);
        long long tw0 = clock64();
        while (!mbar_try_wait(&bar->drain, 0) && clock64() - tw0 < kWaitLimitCycles) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / merge
    // Every tcgen05.ld / st below is warp-collective: the branches around them
    // are warp-uniform, and only the global loads and stores depend on the row.
    // The four warps leave the tile loop together (a barrier that ORs their
    // failures), so none is left at a named barrier. Per tile: P from S, then
    // (while the tensor core forms O) the row's sparse output is fetched and
    // the next tile's biases are built, then the merge.
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int tw = (p.nkb + 31) / 32;
    // biases of tile it into sBias[it % 2]: bias_b = log2 of cluster b's keys
    // outside the tile's computed key tiles (the bitmap of its CSR row)
    auto build_bias = [&](int it) {
      const int u = T0 + it, bh = u / p.nqb, r = u - bh * p.nqb;
      for (int i = tid; i < tw; i += 128) bar->tiles[i] = 0u;
      named_bar_sync(1, 128);
      const int row = bh * p.nqb + r;
      const int c0 = p.row_ptr[row], c1 = p.row_ptr[row + 1];
      for (int i = c0 + tid; i < c1; i += 128) {
        const int t = p.col_idx[i];
        if (t >= 0 && t < p.nkb) atomicOr(&bar->tiles[t >> 5], 1u << (t & 31));
        else atomicOr(p.status, kDevErrBounds);
      }
      named_bar_sync(1, 128);
      const int32_t* off = p.offsets_k + static_cast<size_t>(bh) * (p.C + 1);
      float* bias = sBias + (it & 1) * kMaxC;
      for (int b = tid; b < p.C; b += 128) {
        const int k0 = off[b], k1 = off[b + 1];
        int covered = 0;
        if (k1 > k0) {
          for (int t = k0 / p.bk; t <= (k1 - 1) / p.bk; ++t) {
            if ((bar->tiles[t >> 5] >> (t & 31)) & 1u) {
              const int lo = max(k0, t * p.bk), hi = min(k1, (t + 1) * p.bk);
              covered += hi - lo;
            }
          }
        }
        const int nb = k1 - k0 - covered;
        bias[b] = nb > 0 ? __log2f(static_cast<float>(nb)) : -INFINITY;
      }
      named_bar_sync(1, 128);  // the biases are complete, and the bitmap may be rebuilt
    };
    bool ok = true;
    if (n > 0) build_bias(0);
    for (int it = 0; it < n; ++it) {
      if (named_bar_or(1, 128, !ok || *abort_flag != 0)) break;
      const int u = T0 + it, bh = u / p.nqb, r = u - bh * p.nqb;
      const float* bias = sBias + (it & 1) * kMaxC;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar->s_full, it & 1, abort_flag, p.status));
      float m = -INFINITY, den = 0.0f;
      if (ok) {
        tc_fence_after();
        // S in 32-column chunks, two loads in flight per wait; the C % 32 = 16
        // tail alone
        const int n32 = p.C / 32;
        const float* tail_bias = bias + n32 * 32;
        for (int ch = 0; ch < n32; ch += 2) {
          uint32_t sa[32], sb[32];
          const bool two = ch + 1 < n32;  // warp-uniform
          tmem_ld_32x32b_x32(lane_base + Cf::kColS + ch * 32, sa);
          if (two) tmem_ld_32x32b_x32(lane_base + Cf::kColS + (ch + 1) * 32, sb);
          tmem_ld_wait();
          reg_fence(sa);
          reg_fence(sb);
#pragma unroll
          for (int i = 0; i < 32; ++i) m = fmaxf(m, fmaf(u2f(sa[i]), p.scale_log2, bias[ch * 32 + i]));
          if (two) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              m = fmaxf(m, fmaf(u2f(sb[i]), p.scale_log2, bias[(ch + 1) * 32 + i]));
          }
        }
        if (p.C % 32 != 0) {
          uint32_t s[16];
          tmem_ld_32x32b_x16(lane_base + Cf::kColS + n32 * 32, s);
          tmem_ld_wait();
          reg_fence(s);
#pragma unroll
          for (int i = 0; i < 16; ++i) m = fmaxf(m, fmaf(u2f(s[i]), p.scale_log2, tail_bias[i]));
        }
        const float mu = m == -INFINITY ? 0.0f : m;
        // P: S columns [32 ch, 32 ch + 32) -> P columns [16 ch, 16 ch + 16), which
        // hold S columns already read
        auto exp_chunk = [&](const uint32_t (&s)[32], int ch) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int b = ch * 32 + 2 * i;
            const float p0 = fast_exp2(fmaf(u2f(s[2 * i]), p.scale_log2, bias[b]) - mu);
            const float p1 = fast_exp2(fmaf(u2f(s[2 * i + 1]), p.scale_log2, bias[b + 1]) - mu);
            den += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st_32x32b_x16(lane_base + Cf::kColS + ch * 16, pk);
        };
        for (int ch = 0; ch < n32; ch += 2) {
          uint32_t sa[32], sb[32];
          const bool two = ch + 1 < n32;  // warp-uniform
          tmem_ld_32x32b_x32(lane_base + Cf::kColS + ch * 32, sa);
          if (two) tmem_ld_32x32b_x32(lane_base + Cf::kColS + (ch + 1) * 32, sb);
          tmem_ld_wait();
          reg_fence(sa);
          reg_fence(sb);
          exp_chunk(sa, ch);
          if (two) exp_chunk(sb, ch + 1);
        }
        if (p.C % 32 != 0) {
          uint32_t s[16];
          tmem_ld_32x32b_x16(lane_base + Cf::kColS + n32 * 32, s);
          tmem_ld_wait();
          reg_fence(s);
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float p0 = fast_exp2(fmaf(u2f(s[2 * i]), p.scale_log2, tail_bias[2 * i]) - mu);
            const float p1 =
                fast_exp2(fmaf(u2f(s[2 * i + 1]), p.scale_log2, tail_bias[2 * i + 1]) - mu);
            den += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st_32x32b_x8(lane_base + Cf::kColS + n32 * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar->p_full);
      }
      // this row's sparse output and log-sum-exp, fetched while O is formed
      // (rows past N only take part in the warp's tensor-memory loads)
      const int qrow = r * 128 + tid;
      const bool row_ok = qrow < p.N;
      const size_t ro = static_cast<size_t>(bh) * p.N + (row_ok ? qrow : 0);
      uint4* dst = reinterpret_cast<uint4*>(p.os + ro * D);
      uint4 sp[D / 8];
      float lse2 = -INFINITY;
      if (ok && row_ok) {
#pragma unroll
        for (int i = 0; i < D / 8; ++i) sp[i] = dst[i];
        lse2 = p.lse[ro] * 1.4426950408889634f;
      }
      if (it + 1 < n) build_bias(it + 1);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar->o_full, it & 1, abort_flag, p.status));
      if (!ok) continue;  // leaves at the next iteration's barrier
      tc_fence_after();
      const float M = fmaxf(lse2, m);
      const float a = lse2 == -INFINITY ? 0.0f : fast_exp2(lse2 - M);
      const float c = m == -INFINITY ? 0.0f : fast_exp2(m - M);
      const float tot = a + den * c;
      const float inv = tot > 0.0f ? 1.0f / tot : 0.0f;  // no key at all: O = 0
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(lane_base + Cf::kColO + ch * 32, o);
        tmem_ld_wait();
        reg_fence(o);
        if (!row_ok) continue;
        uint32_t pk[16];
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const uint4 in = sp[ch * 4 + v4];
          const uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int e = 8 * v4 + 2 * i;
            const float s0 = __uint_as_float(w[i] << 16), s1 = __uint_as_float(w[i] & 0xffff0000u);
            pk[4 * v4 + i] = pack_bf16x2((s0 * a + u2f(o[e]) * c) * inv,
                                         (s1 * a + u2f(o[e + 1]) * c) * inv);
          }
        }
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          dst[ch * 4 + v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
      }
      tc_fence_before();
      mbar_arrive(&bar->o_empty);
    }
    if (!ok && tid == 0) atomicOr(p.status, kDevErrTimeout);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t kmeans_workspace_bytes(int32_t BH, int32_t N, int32_t D, int32_t C) {
  const size_t nblk = (static_cast<size_t>(N) + kSortRows - 1) / kSortRows;
  size_t b = 0;
  auto add = [&](size_t n) { b = (b + 255) / 256 * 256 + n; };
  add(static_cast<size_t>(BH) * C * D * 2);        // bf16 centroids
  add(static_cast<size_t>(BH) * C * 4);            // norms
  add(static_cast<size_t>(BH) * nblk * C * 4);     // sort histograms
  add(static_cast<size_t>(BH) * C * D * 4);        // the other centroid buffer
  add(static_cast<size_t>(BH) * ((N + kChunkRows - 1) / kChunkRows + C) * D * 4);  // run sums
  return (b + 255) / 256 * 256;
}

namespace {
struct KWs {
  svg_bf16* cb;
  float* norms;
  int32_t* hist;
  float* cent2;
  float* partial;
};
KWs carve(void* ws, int32_t BH, int32_t N, int32_t D, int32_t C) {
  const size_t nblk = (static_cast<size_t>(N) + kSortRows - 1) / kSortRows;
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t b = 0;
  auto take = [&](size_t n) {
    b = (b + 255) / 256 * 256;
    uint8_t* p = base + b;
    b += n;
    return p;
  };
  KWs w;
  w.cb = reinterpret_cast<svg_bf16*>(take(static_cast<size_t>(BH) * C * D * 2));
  w.norms = reinterpret_cast<float*>(take(static_cast<size_t>(BH) * C * 4));
  w.hist = reinterpret_cast<int32_t*>(take(static_cast<size_t>(BH) * nblk * C * 4));
  w.cent2 = reinterpret_cast<float*>(take(static_cast<size_t>(BH) * C * D * 4));
  w.partial = reinterpret_cast<float*>(
      take(static_cast<size_t>(BH) * ((N + kChunkRows - 1) / kChunkRows + C) * D * 4));
  return w;
}

template <int D>
cudaError_t launch_assign(int32_t BH, int32_t N, int32_t C, const svg_bf16* x, const KWs& w,
                          int32_t* assign, int* status, cudaStream_t stream) {
  using Cf = AsgCfg<D>;
  AsgParams p;
  memset(&p, 0, sizeof(p));
  if (!make_tmap_bf16(&p.tm_x, x, D, N, BH, 128) || !make_tmap_bf16(&p.tm_c, w.cb, D, C, BH, C))
    return cudaErrorInvalidValue;
  p.norms = w.norms;
  p.assign = assign;
  p.status = status;
  p.N = N;
  p.C = C;
  p.n_tiles = (N + 127) / 128;
  // one wave of CTAs over all heads (148 SMs), at least one per head
  int per = 148 / BH;
  if (per > p.n_tiles) per = p.n_tiles;
  if (per < 1) per = 1;
  p.ctas_per_head = per;
  auto kern = kmeans_assign_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(per, BH), kAsgThreads, Cf::kSmem, stream>>>(p);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_kmeans_assign(int32_t BH, int32_t N, int32_t D, int32_t C, const svg_bf16* x,
                                 const float* centroids, int32_t* assign, void* ws, int* status,
                                 cudaStream_t stream) {
  const KWs w = carve(ws, BH, N, D, C);
  const int rows = BH * C;
  kmeans_prep_kernel<<<(rows + 7) / 8, 256, 0, stream>>>(centroids, rows, D, w.cb, w.norms);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return D == 128 ? launch_assign<128>(BH, N, C, x, w, assign, status, stream)
                  : launch_assign<64>(BH, N, C, x, w, assign, status, stream);
}

cudaError_t launch_cluster_sort(int32_t BH, int32_t N, int32_t C, const int32_t* assign,
                                int32_t* order, int32_t* offsets, void* ws, int32_t D, int* status,
                                cudaStream_t stream) {
  const KWs w = carve(ws, BH, N, D, C);
  const int nblk = (N + kSortRows - 1) / kSortRows;
  const size_t sm = static_cast<size_t>(C) * sizeof(int);
  sort_hist_kernel<<<dim3(nblk, BH), 256, sm, stream>>>(assign, N, C, nblk, w.hist, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sort_scan_kernel<<<BH, 256, 0, stream>>>(w.hist, N, C, nblk, offsets);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sort_rank_kernel<<<dim3(nblk, BH), 32, sm, stream>>>(assign, w.hist, N, C, nblk, order);
  return cudaGetLastError();
}

cudaError_t launch_kmeans_update(int32_t BH, int32_t N, int32_t D, int32_t C, const svg_bf16* x,
                                 const int32_t* order, const int32_t* offsets, const float* c_in,
                                 float* c_out, void* ws, int* status, cudaStream_t stream) {
  const KWs w = carve(ws, BH, N, D, C);
  const int nchunks = (N + kChunkRows - 1) / kChunkRows;
  const dim3 g_sum(static_cast<unsigned>((nchunks + kChunkWarps - 1) / kChunkWarps),
                   static_cast<unsigned>(BH));
  const dim3 g_mean(static_cast<unsigned>((C + kChunkWarps - 1) / kChunkWarps),
                    static_cast<unsigned>(BH));
  cudaError_t e;
  if (D == 128) {
    e = cudaFuncSetAttribute(kmeans_chunk_sum_kernel<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ChunkCfg<128>::kSmem);
    if (e != cudaSuccess) return e;
    kmeans_chunk_sum_kernel<128><<<g_sum, 32 * kChunkWarps, ChunkCfg<128>::kSmem, stream>>>(
        x, order, offsets, N, C, nchunks, w.partial, status);
    kmeans_mean_kernel<128><<<g_mean, 32 * kChunkWarps, 0, stream>>>(w.partial, offsets, C,
                                                                     nchunks, c_in, c_out);
  } else {
    e = cudaFuncSetAttribute(kmeans_chunk_sum_kernel<64>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ChunkCfg<64>::kSmem);
    if (e != cudaSuccess) return e;
    kmeans_chunk_sum_kernel<64><<<g_sum, 32 * kChunkWarps, ChunkCfg<64>::kSmem, stream>>>(
        x, order, offsets, N, C, nchunks, w.partial, status);
    kmeans_mean_kernel<64><<<g_mean, 32 * kChunkWarps, 0, stream>>>(w.partial, offsets, C, nchunks,
                                                                    c_in, c_out);
  }
  return cudaGetLastError();
}

cudaError_t launch_kmeans(int32_t BH, int32_t N, int32_t D, int32_t C, int32_t iters,
                          const svg_bf16* x, float* centroids, int32_t* assign, int32_t* order,
                          int32_t* offsets, void* ws, int* status, cudaStream_t stream) {
  const KWs w = carve(ws, BH, N, D, C);
  kmeans_init_kernel<<<dim3(C, BH), 128, 0, stream>>>(x, N, D, C, centroids);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the iterations alternate between the caller's buffer and the workspace
  // copy so that the last update lands in the caller's buffer
  float* bufs[2] = {centroids, w.cent2};
  int cur = 0;
  if (iters % 2 == 1) {
    e = cudaMemcpyAsync(w.cent2, centroids, static_cast<size_t>(BH) * C * D * 4,
                        cudaMemcpyDeviceToDevice, stream);
    if (e != cudaSuccess) return e;
    cur = 1;
  }
  for (int it = 0; it < iters; ++it) {
    if ((e = launch_kmeans_assign(BH, N, D, C, x, bufs[cur], assign, ws, status, stream)) !=
        cudaSuccess)
      return e;
    if ((e = launch_cluster_sort(BH, N, C, assign, order, offsets, ws, D, status, stream)) !=
        cudaSuccess)
      return e;
    if ((e = launch_kmeans_update(BH, N, D, C, x, order, offsets, bufs[cur], bufs[cur ^ 1], ws,
                                  status, stream)) != cudaSuccess)
      return e;
    cur ^= 1;
  }
  if (iters == 0) {
    if ((e = launch_kmeans_assign(BH, N, D, C, x, centroids, assign, ws, status, stream)) !=
        cudaSuccess)
      return e;
    return launch_cluster_sort(BH, N, C, assign, order, offsets, ws, D, status, stream);
  }
  return cudaSuccess;
}

cudaError_t launch_select_clusters(int32_t BH, int32_t D, int32_t Cq, int32_t Ck, float scale,
                                   float top_p, const float* cq, const float* ck,
                                   const int32_t* offsets_k, const float* disp, float tau,
                                   uint32_t* sel, cudaStream_t stream) {
  const int threads = (Ck + 31) / 32 * 32;
  const size_t sm = static_cast<size_t>(kSelGroup) * (Ck + 32 + D) * sizeof(float);
  if (sm > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sm));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((Cq + kSelGroup - 1) / kSelGroup), static_cast<unsigned>(BH));
  select_kernel<<<grid, threads, sm, stream>>>(cq, ck, offsets_k, D, Cq, Ck, scale, top_p, disp,
                                               tau, sel);
  return cudaGetLastError();
}

cudaError_t launch_tile_csr(int32_t BH, int32_t N, int32_t Cq, int32_t Ck, int32_t bq, int32_t bk,
                            const int32_t* offsets_q, const int32_t* offsets_k, const uint32_t* sel,
                            int32_t* row_ptr, int32_t* col_idx, int64_t capacity, int32_t* counts,
                            int* status, cudaStream_t stream) {
  const int nqb = (N + bq - 1) / bq, nkb = (N + bk - 1) / bk;
  const int rows = BH * nqb;
  const int blocks = (rows + kTileWarps - 1) / kTileWarps;
  tile_count_kernel<<<blocks, 32 * kTileWarps, 0, stream>>>(offsets_q, offsets_k, sel, BH, N, Cq,
                                                            Ck, bq, bk, nqb, nkb, counts);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  tile_scan_kernel<<<1, 1024, 0, stream>>>(counts, rows, row_ptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  tile_fill_kernel<<<blocks, 32 * kTileWarps, 0, stream>>>(offsets_q, offsets_k, sel, BH, N, Cq, Ck,
                                                           bq, bk, nqb, nkb, row_ptr, col_idx,
                                                           capacity, status);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows(int32_t BH, int32_t N, int32_t D, const svg_bf16* x,
                                const int32_t* order, svg_bf16* y, bool scatter, int* status,
                                cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(BH) * N * (D / 8);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 16 * 148) blocks = 16 * 148;
  if (scatter)
    permute_rows_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(x, order, BH, N, D,
                                                                                 y, status);
  else
    permute_rows_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(x, order, BH, N,
                                                                                  D, y, status);
  return cudaGetLastError();
}

}  // namespace svg

namespace svg {

cudaError_t launch_cluster_stats(int32_t BH, int32_t N, int32_t D, int32_t C, const svg_bf16* v,
                                 const int32_t* order, const int32_t* offsets, float* vbar,
                                 float* disp, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(C), static_cast<unsigned>(BH));
  if (D == 128)
    cluster_stats_kernel<128><<<grid, 32 * kSumWarps, 0, stream>>>(v, order, offsets, N, C, vbar,
                                                                   disp);
  else
    cluster_stats_kernel<64><<<grid, 32 * kSumWarps, 0, stream>>>(v, order, offsets, N, C, vbar,
                                                                  disp);
  return cudaGetLastError();
}

size_t ear_workspace_bytes(int32_t BH, int32_t D, int32_t C) {
  return (static_cast<size_t>(BH) * C * D * 2 * 2 + 255) / 256 * 256;
}

cudaError_t launch_ear_compensate(int32_t BH, int32_t N, int32_t D, int32_t C, int32_t bk,
                                  float scale, const svg_bf16* qs, const float* kbar,
                                  const float* vbar, const int32_t* offsets_k,
                                  const int32_t* row_ptr, const int32_t* col_idx, svg_bf16* os,
                                  const float* lse, void* ws, int* status, cudaStream_t stream) {
  svg_bf16* kb = static_cast<svg_bf16*>(ws);
  svg_bf16* vb = kb + static_cast<size_t>(BH) * C * D;
  const int64_t n = static_cast<int64_t>(BH) * C * D;
  to_bf16_kernel<<<static_cast<unsigned>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0,
                   stream>>>(kbar, n, kb);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  to_bf16_kernel<<<static_cast<unsigned>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0,
                   stream>>>(vbar, n, vb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  EarParams p;
  memset(&p, 0, sizeof(p));
  if (!make_tmap_bf16(&p.tm_q, qs, D, N, BH, 128) || !make_tmap_bf16(&p.tm_kb, kb, D, C, BH, C) ||
      !make_tmap_bf16(&p.tm_vb, vb, D, C, BH, C))
    return cudaErrorInvalidValue;
  p.offsets_k = offsets_k;
  p.row_ptr = row_ptr;
  p.col_idx = col_idx;
  p.os = os;
  p.lse = lse;
  p.status = status;
  p.N = N;
  p.C = C;
  p.bk = bk;
  p.BH = BH;
  p.nqb = (N + 127) / 128;
  p.nkb = (N + bk - 1) / bk;
  p.scale_log2 = scale * 1.4426950408889634f;
  // persistent: one CTA per SM (each takes all tensor-memory columns)
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const long long tiles = static_cast<long long>(BH) * p.nqb;
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
  if (D == 128) {
    auto kern = ear_compensate_kernel<128>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  EarCfg<128>::kSmem)) != cudaSuccess)
      return e;
    kern<<<grid, kEarThreads, EarCfg<128>::kSmem, stream>>>(p);
  } else {
    auto kern = ear_compensate_kernel<64>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  EarCfg<64>::kSmem)) != cudaSuccess)
      return e;
    kern<<<grid, kEarThreads, EarCfg<64>::kSmem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace svg
