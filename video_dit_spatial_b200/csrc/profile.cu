// Online profiling of Sparse VideoGen (arXiv 2502.01776 abstract: "an online
// profiling strategy to capture the dynamic sparse patterns and predict the
// type of attention head"). For sampled query rows of every head, full
// attention is compared with spatial-masked and temporal-masked attention by
// the mean squared error of the outputs; the mask with the smaller error names
// the head's type.
//
// One CTA = one (b*H + h, tile of 128 sampled rows). It runs flash attention of
// its 128 gathered query rows over ALL keys (64-key tiles, TMA-fed) and keeps
// three online softmaxes side by side: the full one and the two token-level
// masked ones, each with its own running maximum. The exponentials are taken
// once, for the full softmax; each masked probability is the full one times
// 2^(m_full - m_mask) on the keys its mask allows.
//
// 320 threads: warps 0-7 softmax, warp 8 TMA producer, warp 9 MMA issuer.
// Warps w and w+4 own the same 32 query rows (TMEM lanes 32*(w%4)..+31) and
// split each 64-key tile into keys [0,32) and [32,64); they exchange row maxima
// through shared memory (one 64-thread named barrier per warp pair) and keep
// partial row sums that are added once at the end.
// Tensor memory: S double buffer (64 columns each at 0 and 64), O_full (128),
// O_spatial (128 + d), O_temporal (128 + 2d). P_full and P_temporal (bf16)
// overwrite the two halves of their S buffer and feed their PV products from
// tensor memory; P_spatial goes to a double-buffered swizzled tile in shared
// memory and feeds its product from there. A masked product is skipped for key
// tiles where no row of the CTA has an allowed key, and a warp rewrites its
// rows of a P_spatial buffer only when they are not already zero. The allowed keys of a row
// inside a tile are at most a few index runs (spatial: the frames [f-s, f+s];
// temporal: positions [p-w, p+w] of each frame; text keys always), built as
// bit ranges. Each CTA reduces sum((O_X - O_full)^2) over its rows in a fixed
// order into the workspace; a second kernel adds the tiles in a fixed order
// and labels the head.
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace svg {
namespace {

constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = (kSoftmaxWarps + 2) * 32;
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;
constexpr int kRows = 128;  // sampled rows per CTA
constexpr int kKeys = 64;   // keys per tile
constexpr int kHalf = 32;   // keys per softmax thread per tile
constexpr int kKStages = 4;
constexpr int kVStages = 3;
constexpr float kRebaseLog2 = 8.0f;

struct PBarriers {
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_full, o_final, drain;
  uint32_t tmem_base;
  int abort_flag;
  int x_active[2][2][kSoftmaxWarps];  // [buffer][mask][warp]
  float xmax[2][3][kRows];            // [half][full, spatial, temporal][row]
  float xsum[2][3][kRows];            // [half][full, spatial, temporal][row]
  float red[2][2][kRows];             // [half][spatial, temporal][row]
  int pair_fail[4][2];
};

template <int D>
struct PCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kQPanel = kRows * 128;   // 128 rows x 128 B
  static constexpr int kKVPanel = kKeys * 128;  // 64 rows x 128 B
  static constexpr int kQBytes = kPanels * kQPanel;
  static constexpr int kKVBytes = kPanels * kKVPanel;
  static constexpr int kPBytes = kRows * kKeys * 2;  // one masked P tile, K-major swizzled
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  static constexpr int kOffP = kOffV + kVStages * kKVBytes;  // P_spatial [buffer]
  static constexpr int kOffBar = kOffP + 2 * kPBytes;
  static constexpr int kBarBytes = (static_cast<int>(sizeof(PBarriers)) + 127) / 128 * 128;
  static constexpr int kUsed = kOffBar + kBarBytes + 1024;
  static constexpr int kSmem = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 64;
  static constexpr uint32_t kColOF = 128, kColOS = 128 + D, kColOT = 128 + 2 * D;
  static_assert(kColOT + D <= kTmemCols, "accumulators must fit tensor memory");
  static_assert(kOffP % 1024 == 0, "swizzled tiles start on 1024-byte boundaries");
  static_assert(kOffBar + kBarBytes + 1024 <= kSmem, "bookkeeping must fit the allocation");
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
};

// With n_splits > 1 each (head, sample tile) runs as n_splits CTAs over
// consecutive ranges of key tiles; each writes its unnormalised accumulators
// and (base, sum) pairs, and profile_combine_kernel merges them.
struct __align__(64) ProfParams {
  CUtensorMap tm_k, tm_v;
  const svg_bf16* q;
  const int32_t* sample_idx;
  float* partial;  // [BH][2][n_tiles]
  float* part_o;   // [BH][n_tiles][n_splits][3][D][128] (n_splits > 1)
  float* part_ml;  // [BH][n_tiles][n_splits][3][2][128] (n_splits > 1)
  int* status;
  int32_t n_samples, n_tiles, n_splits;
  int32_t N, Nv, T, P, s, w, nkt;
  float scale_log2;
};


__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// Barrier of the two warps that share a group of 32 rows (ids 1..4).
__device__ __forceinline__ void pair_sync(int group) {
  asm volatile("bar.sync %0, 64;" ::"r"(1 + group) : "memory");
}

__device__ __forceinline__ void softmax_sync() {
  asm volatile("bar.sync 5, 256;" ::: "memory");
}

// Bits [a, b) of a 32-bit word, for 0 <= a, b <= 32 (empty when b <= a).
__device__ __forceinline__ uint32_t bit_range32(int a, int b) {
  a = max(a, 0);
  b = min(b, 32);
  if (b <= a) return 0u;
  return static_cast<uint32_t>((1ull << b) - (1ull << a));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Masked probabilities of one half tile for one mask, from the full ones.
//   SHAPE 0: some keys allowed (per-key selection), 1: no key allowed in the
//   warp, 2: every key allowed in the warp, 3: the masked base is far below the
//   full one for some row, so allowed keys take their own exponential.
template <int SHAPE>
__device__ __forceinline__ void masked_pass(const float (&f)[kHalf], const uint32_t (&sr)[kHalf],
                                            uint32_t bits, float k, bool direct, float scale_log2,
                                            float u, uint32_t (&pk)[kHalf / 2], float& sum) {
  float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
  for (int i = 0; i < kHalf / 2; ++i) {
    float g0, g1;
    if (SHAPE == 1) {
      g0 = g1 = 0.0f;
    } else {
      ffma2(g0, g1, f[2 * i], f[2 * i + 1], k, k, 0.0f, 0.0f);
      if (SHAPE == 3 && direct) {
        g0 = fast_exp2(fmaf(u2f(sr[2 * i]), scale_log2, -u));
        g1 = fast_exp2(fmaf(u2f(sr[2 * i + 1]), scale_log2, -u));
      }
      if (SHAPE != 2) {
        g0 = (bits >> (2 * i)) & 1u ? g0 : 0.0f;
        g1 = (bits >> (2 * i + 1)) & 1u ? g1 : 0.0f;
      }
      fadd2(s0, s1, s0, s1, g0, g1);
    }
    pk[i] = pack_bf16x2(g0, g1);
  }
  sum = s0 + s1;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) profile_kernel(const __grid_constant__ ProfParams p) {
  using C = PCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sP = smem + C::kOffP;
  PBarriers* bar = reinterpret_cast<PBarriers*>(smem + C::kOffBar);
  volatile int* abort_flag = &bar->abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int tile = blockIdx.x;
  const int bh = blockIdx.y;
  // this CTA's key tiles: [j0, j0 + n)
  const int split = blockIdx.z;
  const int j0 = static_cast<int>(static_cast<long long>(p.nkt) * split / p.n_splits);
  const int n = static_cast<int>(static_cast<long long>(p.nkt) * (split + 1) / p.n_splits) - j0;

  if (warp == 0) {
    tmem_alloc(&bar->tmem_base, C::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 32) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->p_full[s], 32 * kSoftmaxWarps);
    }
    mbar_init(&bar->o_full, 1);
    mbar_init(&bar->o_final, 1);
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_mbar_init();
  }
  // Gather the sampled Q rows into the swizzled K-major tile: row r = tid % 128,
  // half h = tid / 128 copies 16-byte chunks [h*D/16, (h+1)*D/16). Rows past the
  // sample count, and out-of-range indices, become zero rows.
  const int row = tid & 127;
  const int half = (tid >> 7) & 1;
  int qrow = -1;
  if (warp < kSoftmaxWarps) {
    const int si = tile * kRows + row;
    if (si < p.n_samples) {
      const int r = __ldg(p.sample_idx + si);
      if (r >= 0 && r < p.Nv) {
        qrow = r;
      } else if (half == 0) {
        atomicOr(p.status, kDevErrBounds);
      }
    }
    const uint4* src = reinterpret_cast<const uint4*>(
        p.q + (static_cast<size_t>(bh) * p.N + (qrow >= 0 ? qrow : 0)) * D);
#pragma unroll
    for (int cc = 0; cc < D / 16; ++cc) {
      const int c = half * (D / 16) + cc;
      const uint4 v = qrow >= 0 ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
      const int pn = c >> 3, ci = c & 7;
      *reinterpret_cast<uint4*>(sQ + pn * C::kQPanel + row * 128 + ((ci ^ (row & 7)) << 4)) = v;
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;

  if (warp == kProducerWarp) {
    if (lane_id() == 0) {
      const uint64_t keep = l2_policy_evict_last();
      // K runs up to kKStages tiles ahead, V up to kVStages; K(j) is issued
      // before V(j-1) so the deeper K ring is used.
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          const int st = j % kKStages;
          ok = mbar_wait(&bar->k_empty[st], ((j / kKStages) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          mbar_arrive_expect_tx(&bar->k_full[st], C::kKVBytes);
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d_hint(sK + st * C::kKVBytes + pn * C::kKVPanel, &p.tm_k, &bar->k_full[st],
                             pn * 64, (j0 + j) * kKeys, bh, keep);
          k_issued = j + 1;
        }
        if (j >= 1) {
          const int jv = j - 1;
          const int st = jv % kVStages;
          ok = mbar_wait(&bar->v_empty[st], ((jv / kVStages) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          mbar_arrive_expect_tx(&bar->v_full[st], C::kKVBytes);
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d_hint(sV + st * C::kKVBytes + pn * C::kKVPanel, &p.tm_v, &bar->v_full[st],
                             pn * 64, (j0 + jv) * kKeys, bh, keep);
          v_issued = jv + 1;
        }
      }
      if (*abort_flag) {
        // Let every copy this thread started land before the CTA retires.
        for (int j = (k_issued > kKStages ? k_issued - kKStages : 0); j < k_issued; ++j) {
          long long t0 = clock64();
          while (!mbar_try_wait(&bar->k_full[j % kKStages], (j / kKStages) & 1) &&
                 clock64() - t0 < kWaitLimitCycles) {
          }
        }
        for (int j = (v_issued > kVStages ? v_issued - kVStages : 0); j < v_issued; ++j) {
          long long t0 = clock64();
          while (!mbar_try_wait(&bar->v_full[j % kVStages], (j / kVStages) & 1) &&
                 clock64() - t0 < kWaitLimitCycles) {
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane_id() == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kKeys, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      const uint32_t p_addr = smem_u32(sP);
      bool started[2] = {false, false};
      for (int j = 0; j <= n; ++j) {
        if (j < n) {
          const int st = j % kKStages;
          const uint32_t s_col = tmem + ((j & 1) ? C::kColS1 : C::kColS0);
          if (!mbar_wait(&bar->k_full[st], (j / kKStages) & 1, abort_flag, p.status)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            mma_bf16_ss(s_col, sdesc_sw128(q_addr + (kk >> 2) * C::kQPanel + off, 16, 1024),
                        sdesc_sw128(k_addr + st * C::kKVBytes + (kk >> 2) * C::kKVPanel + off, 16,
                                    1024),
                        idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc_commit(&bar->s_full[j & 1]);
          tc_commit(&bar->k_empty[st]);  // K(j) is free once QK_j retires
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj % kVStages;
          const int sb = jj & 1;
          const uint32_t pf_col = tmem + (sb ? C::kColS1 : C::kColS0);
          if (!mbar_wait(&bar->p_full[sb], (jj >> 1) & 1, abort_flag, p.status)) break;
          if (!mbar_wait(&bar->v_full[st], (jj / kVStages) & 1, abort_flag, p.status)) break;
          tc_fence_after();
          int active[2] = {0, 0};
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const volatile int* xa = bar->x_active[sb][m];
#pragma unroll
            for (int w = 0; w < kSoftmaxWarps; ++w) active[m] |= xa[w];
          }
          const uint32_t vb = v_addr + st * C::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk)
            mma_bf16_ts(tmem + C::kColOF, pf_col + kk * 8,
                        sdesc_sw128(vb + kk * 16 * 128, C::kKVPanel, 1024), idesc_pv,
                        (jj > 0 || kk > 0) ? 1u : 0u);
          if (active[0]) {  // spatial: P from shared memory
            const uint32_t pm = p_addr + sb * C::kPBytes;
#pragma unroll
            for (int kk = 0; kk < kKeys / 16; ++kk)
              mma_bf16_ss(tmem + C::kColOS, sdesc_sw128(pm + kk * 32, 16, 1024),
                          sdesc_sw128(vb + kk * 16 * 128, C::kKVPanel, 1024), idesc_pv,
                          (started[0] || kk > 0) ? 1u : 0u);
            started[0] = true;
          }
          if (active[1]) {  // temporal: P from the upper half of the S buffer
#pragma unroll
            for (int kk = 0; kk < kKeys / 16; ++kk)
              mma_bf16_ts(tmem + C::kColOT, pf_col + kKeys / 2 + kk * 8,
                          sdesc_sw128(vb + kk * 16 * 128, C::kKVPanel, 1024), idesc_pv,
                          (started[1] || kk > 0) ? 1u : 0u);
            started[1] = true;
          }
          tc_commit(&bar->v_empty[st]);
          tc_commit(&bar->o_full);
          if (jj == n - 1) tc_commit(&bar->o_final);
        }
      }
      if (*abort_flag) {
        tc_commit(&bar->drain);
        long long t0 = clock64();
        while (!mbar_try_wait(&bar->drain, 0) && clock64() - t0 < kWaitLimitCycles) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int group = warp & 3;       // rows 32*group .. +31 (TMEM lane quarter)
    const int c_base = half * kHalf;  // this thread's key columns within a tile
    const bool row_valid = qrow >= 0;
    const int qi = row_valid ? qrow : 0;
    const int f_i = qi / p.P;
    const int p_i = qi - f_i * p.P;
    // Allowed video keys of this row: spatial = the frames [f_i - s, f_i + s]
    // (one index run); temporal = positions [p_i - w, p_i + w] of every frame
    // (one run per frame). Text keys [Nv, N) are allowed by both.
    const int s_lo = max(f_i - p.s, 0) * p.P;
    const int s_hi = static_cast<int>(min(static_cast<long long>(f_i) + p.s + 1,
                                          static_cast<long long>(p.T))) * p.P;
    const int t_lo = max(p_i - p.w, 0);
    const int t_hi = static_cast<int>(
        min(static_cast<long long>(p_i) + p.w, static_cast<long long>(p.P - 1)));
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(group * 32) << 16);
    const uint32_t p_row = smem_u32(sP) + row * 128;
    // running bases (log2 units) and sums of the full, spatial, temporal softmax
    float m[3] = {-INFINITY, -INFINITY, -INFINITY};
    float l[3] = {0.0f, 0.0f, 0.0f};
    bool ok = true;
    // start of the frame holding this thread's first key of the tile
    // Allowed-key bits of a half tile: text keys, the spatial run, and the
    // temporal run of each frame overlapping the half tile. r0 = k0 mod P; with
    // P >= 32 at most two frames overlap 32 keys and the bits need no branch,
    // so the next tile's bits are computed in the shadow of this tile's
    // exponentials.
    auto tile_bits = [&](int jt, int r0, uint32_t (&b)[2]) {
      const int k0 = (j0 + jt) * kKeys + c_base;
      const int kvalid = max(0, min(kHalf, p.N - k0));
      const int v_end = min(k0 + kvalid, p.Nv);
      const uint32_t text = bit_range32(p.Nv - k0, kvalid);
      uint32_t bt = 0u;
      if (p.P >= kHalf) {
        const int fs = k0 - r0;
        bt = bit_range32(fs + t_lo - k0, min(fs + t_hi + 1, v_end) - k0) |
             bit_range32(fs + p.P + t_lo - k0, min(fs + p.P + t_hi + 1, v_end) - k0);
      } else {
        for (int fs = k0 - r0; fs < v_end; fs += p.P)
          bt |= bit_range32(fs + t_lo - k0, min(fs + t_hi + 1, v_end) - k0);
      }
      const bool any = row_valid && kvalid > 0;
      b[0] = any ? text | bit_range32(s_lo - k0, min(s_hi, v_end) - k0) : 0u;
      b[1] = any ? text | bt : 0u;
    };
    auto next_r0 = [&](int r0) {  // (k0 + 64) mod P from k0 mod P
      r0 += kKeys;
      if (p.P >= kKeys / 2) {
        r0 = r0 >= p.P ? r0 - p.P : r0;
        r0 = r0 >= p.P ? r0 - p.P : r0;
      } else {
        r0 %= p.P;
      }
      return r0;
    };
    int r0 = (j0 * kKeys + c_base) % p.P;
    uint32_t bits[2];  // allowed keys k0 + [0, 32) of this tile: spatial, temporal
    tile_bits(0, r0, bits);
    bool ps_zero[2] = {false, false};  // this warp's rows of P_spatial[buffer] hold zeros
    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      const uint32_t s_col = lane_base + (sb ? C::kColS1 : C::kColS0);
      const int k0 = (j0 + j) * kKeys + c_base;  // first key of this thread's half
      const int kvalid = max(0, min(kHalf, p.N - k0));

      if (ok && !mbar_wait(&bar->s_full[sb], (j >> 1) & 1, abort_flag, p.status)) ok = false;
      // Both warps of a pair must take the same path through pair_sync (an
      // unbounded barrier), so they agree on leaving the loop through it.
      if (__any_sync(0xffffffffu, !ok)) ok = false;
      if (lane_id() == 0) bar->pair_fail[group][half] = ok ? 0 : 1;
      float a0 = -INFINITY, a1 = -INFINITY;
      float bmax[2] = {-INFINITY, -INFINITY};
      uint32_t sr[kHalf];
      if (ok) {
        tc_fence_after();
        tmem_ld_32x32b_x32(s_col + c_base, sr);
        tmem_ld_wait();
        reg_fence(sr);
        if (kvalid < kHalf) {  // only the last tile is ragged
#pragma unroll
          for (int c = 0; c < kHalf; ++c)
            if (c >= kvalid) sr[c] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int c = 0; c < kHalf; c += 4) {
          a0 = fmax3(a0, u2f(sr[c]), u2f(sr[c + 1]));
          a1 = fmax3(a1, u2f(sr[c + 2]), u2f(sr[c + 3]));
        }
        // A masked maximum of this half can only move its masked base when the
        // half's full maximum exceeds that base + 2^8; otherwise report -inf:
        // the combined decision and the new base are unchanged.
        const float hmax = fmaxf(a0, a1) * p.scale_log2;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const bool need = bits[x] != 0u && hmax > m[1 + x] + kRebaseLog2;
          if (__any_sync(0xffffffffu, need)) {
            float b0 = -INFINITY, b1 = -INFINITY;
#pragma unroll
            for (int c = 0; c < kHalf; c += 2) {
              b0 = fmaxf(b0, (bits[x] >> c) & 1u ? u2f(sr[c]) : -INFINITY);
              b1 = fmaxf(b1, (bits[x] >> (c + 1)) & 1u ? u2f(sr[c + 1]) : -INFINITY);
            }
            bmax[x] = fmaxf(b0, b1);
          }
        }
      }
      // exchange the half-row maxima with the partner warp
      bar->xmax[half][0][row] = fmaxf(a0, a1);
      bar->xmax[half][1][row] = bmax[0];
      bar->xmax[half][2][row] = bmax[1];
      pair_sync(group);
      float t[3];
#pragma unroll
      for (int x = 0; x < 3; ++x)
        t[x] = fmaxf(bar->xmax[0][x][row], bar->xmax[1][x][row]) * p.scale_log2;
      const int pair_failed = bar->pair_fail[group][0] | bar->pair_fail[group][1];
      pair_sync(group);  // the exchange slots are rewritten next tile
      if (pair_failed) {
        ok = false;
        break;
      }

      bool rb[3];
      float m_new[3], alpha[3], u[3];
#pragma unroll
      for (int x = 0; x < 3; ++x) {
        rb[x] = t[x] > m[x] + kRebaseLog2;
        m_new[x] = rb[x] ? t[x] : m[x];
        alpha[x] = rb[x] ? fast_exp2(m[x] - m_new[x]) : 1.0f;  // exp2(-inf) = 0
        u[x] = m_new[x] == -INFINITY ? 0.0f : m_new[x];
      }
      // full probabilities of this half tile
      float f[kHalf];
      uint32_t pkF[kHalf / 2];
      float sF0 = 0.0f, sF1 = 0.0f;
#pragma unroll
      for (int i = 0; i < kHalf / 2; ++i) {
        float y0, y1;
        ffma2(y0, y1, u2f(sr[2 * i]), u2f(sr[2 * i + 1]), p.scale_log2, p.scale_log2, -u[0],
              -u[0]);
        f[2 * i] = fast_exp2(y0);
        f[2 * i + 1] = fast_exp2(y1);
        fadd2(sF0, sF1, sF0, sF1, f[2 * i], f[2 * i + 1]);
        pkF[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
      }
      tmem_st_32x32b_x16(s_col + half * (kHalf / 2), pkF);
      float sum[3] = {sF0 + sF1, 0.0f, 0.0f};
      uint32_t next_bits[2];
      const int r0_next = next_r0(r0);
      tile_bits(j + 1, r0_next, next_bits);
      // masked probabilities: P_X = P_full * 2^(u_full - u_X) on allowed keys,
      // unless the masked base is so far below the full one that the full
      // probabilities could flush to zero; those rows (rare) take the masked
      // exponentials directly. (With no allowed key seen yet, m_X is -inf and
      // every P_X is zero.)
      int warp_any[2];
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const float gap = u[0] - u[1 + x];
        const bool direct = m_new[1 + x] != -INFINITY && gap > 64.0f;
        const float kx = direct ? 0.0f : fast_exp2(gap);
        const bool w_none = __all_sync(0xffffffffu, bits[x] == 0u);
        const bool w_all = __all_sync(0xffffffffu, bits[x] == 0xffffffffu);
        const bool w_direct = __any_sync(0xffffffffu, direct);
        warp_any[x] = w_none ? 0 : 1;
        uint32_t pk[kHalf / 2];
        if (w_direct)
          masked_pass<3>(f, sr, bits[x], kx, direct, p.scale_log2, u[1 + x], pk, sum[1 + x]);
        else if (w_none)
          masked_pass<1>(f, sr, bits[x], kx, direct, p.scale_log2, u[1 + x], pk, sum[1 + x]);
        else if (w_all)
          masked_pass<2>(f, sr, bits[x], kx, direct, p.scale_log2, u[1 + x], pk, sum[1 + x]);
        else
          masked_pass<0>(f, sr, bits[x], kx, direct, p.scale_log2, u[1 + x], pk, sum[1 + x]);
        if (x == 1) {
          // temporal: keys k -> column 32 + k/2 of the S buffer (its upper half)
          tmem_st_32x32b_x16(s_col + kKeys / 2 + half * (kHalf / 2), pk);
        } else if (!(w_none && ps_zero[sb])) {
          // spatial: this row's 32 keys = chunks 4*half .. 4*half+3 of its
          // 128-byte row in the shared-memory tile
          const uint32_t base = p_row + sb * C::kPBytes;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int chunk = 4 * half + c;
            st_shared_v4(base + ((chunk ^ (row & 7)) << 4), pk[4 * c], pk[4 * c + 1],
                         pk[4 * c + 2], pk[4 * c + 3]);
          }
          ps_zero[sb] = w_none;
        }
      }
      fence_proxy_async_smem();
#pragma unroll
      for (int x = 0; x < 3; ++x) {
        l[x] = l[x] * alpha[x] + sum[x];
        m[x] = m_new[x];
      }
      tmem_st_wait();
      if (lane_id() == 0) {
        bar->x_active[sb][0][warp] = warp_any[0];
        bar->x_active[sb][1][warp] = warp_any[1];
      }

      // Re-base this half's columns of the moved accumulators once PV_{j-1}
      // has landed.
      bool wrb[3];
#pragma unroll
      for (int x = 0; x < 3; ++x) wrb[x] = __any_sync(0xffffffffu, rb[x]);
      if (j > 0 && (wrb[0] || wrb[1] || wrb[2])) {
        // A failed wait is reported through the pair exchange of the next tile.
        if (!mbar_wait(&bar->o_full, (j - 1) & 1, abort_flag, p.status)) ok = false;
        tc_fence_after();
#pragma unroll
        for (int x = 0; x < 3 && ok; ++x) {
          if (!wrb[x]) continue;
          const uint32_t ocol =
              lane_base + (x == 0 ? C::kColOF : (x == 1 ? C::kColOS : C::kColOT)) + half * (D / 2);
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(ocol + ch * 32, o);
            tmem_ld_wait();
            reg_fence(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(u2f(o[i]) * alpha[x]);
            tmem_st_32x32b_x32(ocol + ch * 32, o);
          }
        }
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&bar->p_full[sb]);
      bits[0] = next_bits[0];
      bits[1] = next_bits[1];
      r0 = r0_next;
    }

    // ---- per-row squared errors over this half's d/2 channels
#pragma unroll
    for (int x = 0; x < 3; ++x) bar->xsum[half][x][row] = l[x];
    if (ok && n > 0) ok = mbar_wait(&bar->o_final, 0, abort_flag, p.status);
    softmax_sync();
    if (p.n_splits > 1) {
      // Partial results of this key range: the accumulators as they stand
      // (relative to the running bases) and each row's (base, sum) pairs. A
      // failure anywhere in the CTA turns all its pairs into NaN.
      if (!__all_sync(0xffffffffu, ok)) atomicOr(&bar->abort_flag, 1);
      softmax_sync();
      tc_fence_after();
      const bool all_ok = *abort_flag == 0;
      const size_t cta = (static_cast<size_t>(bh) * p.n_tiles + tile) * p.n_splits + split;
      float* po = p.part_o + cta * 3 * D * kRows;
#pragma unroll
      for (int x = 0; x < 3; ++x) {
        const uint32_t ocol =
            lane_base + (x == 0 ? C::kColOF : (x == 1 ? C::kColOS : C::kColOT)) + half * (D / 2);
#pragma unroll
        for (int ch = 0; ch < D / 64; ++ch) {
          uint32_t o[32];
          if (all_ok && n > 0) {
            tmem_ld_32x32b_x32(ocol + ch * 32, o);
            tmem_ld_wait();
            reg_fence(o);
          }
          const int c0 = half * (D / 2) + ch * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            po[(static_cast<size_t>(x) * D + c0 + i) * kRows + row] =
                all_ok && n > 0 && bar->xsum[0][x][row] + bar->xsum[1][x][row] > 0.0f
                    ? u2f(o[i])
                    : 0.0f;
        }
        if (half == 0) {
          float* pml = p.part_ml + (cta * 3 + x) * 2 * kRows;
          const float L = bar->xsum[0][x][row] + bar->xsum[1][x][row];
          pml[row] = all_ok ? (L > 0.0f ? m[x] : -INFINITY) : __int_as_float(0x7fc00000);
          pml[kRows + row] = all_ok ? L : __int_as_float(0x7fc00000);
        }
      }
    } else {
    float inv[3];
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      const float L = bar->xsum[0][x][row] + bar->xsum[1][x][row];
      inv[x] = L > 0.0f ? 1.0f / L : 0.0f;
    }
    tc_fence_after();
    float err[2] = {0.0f, 0.0f};
    const bool all_ok = __all_sync(0xffffffffu, ok);
    if (all_ok && n > 0) {
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch) {
        uint32_t oF[32], oX[32];
        tmem_ld_32x32b_x32(lane_base + C::kColOF + half * (D / 2) + ch * 32, oF);
        tmem_ld_wait();
        reg_fence(oF);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          tmem_ld_32x32b_x32(lane_base + (x == 0 ? C::kColOS : C::kColOT) + half * (D / 2) +
                                 ch * 32,
                             oX);
          tmem_ld_wait();
          reg_fence(oX);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float ox = inv[1 + x] > 0.0f ? u2f(oX[i]) * inv[1 + x] : 0.0f;
            const float dlt = ox - u2f(oF[i]) * inv[0];
            err[x] = fmaf(dlt, dlt, err[x]);
          }
        }
      }
    }
    bar->red[half][0][row] = row_valid ? err[0] : 0.0f;
    bar->red[half][1][row] = row_valid ? err[1] : 0.0f;
    if (!all_ok) atomicOr(&bar->abort_flag, 1);
    softmax_sync();
    if (tid < 2) {
      const int x = tid;
      float acc = 0.0f;
      for (int i = 0; i < kRows; ++i) acc += bar->red[0][x][i] + bar->red[1][x][i];
      p.partial[(static_cast<size_t>(bh) * 2 + x) * p.n_tiles + tile] =
          *abort_flag ? __int_as_float(0x7fc00000) : acc;
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Merges the key-range partials of one (head, sample tile): per row and
// softmax, weights 2^(m_s - max m) put the splits on one base; the merged
// outputs give the row's squared errors, which are added over rows in a fixed
// order into the same per-tile slot the unsplit kernel fills.
constexpr int kCombineQuarters = 4;  // threads per row, each a quarter of the channels
constexpr int kMaxSplits = 4;

template <int D>
__global__ void __launch_bounds__(kRows * kCombineQuarters)
    profile_combine_kernel(const __grid_constant__ ProfParams p) {
  __shared__ float red[2][kCombineQuarters][kRows];
  const int tile = blockIdx.x, bh = blockIdx.y;
  const int row = threadIdx.x % kRows, quarter = threadIdx.x / kRows;
  const int S = p.n_splits;
  const size_t cta0 = (static_cast<size_t>(bh) * p.n_tiles + tile) * S;
  const int si = tile * kRows + row;
  bool valid = si < p.n_samples;
  if (valid) {
    const int r = __ldg(p.sample_idx + si);
    valid = r >= 0 && r < p.Nv;
  }
  // per split and softmax: weight 2^(m_s - max m) of the split's accumulator
  float m_s[kMaxSplits][3], l_s[kMaxSplits][3];
  bool aborted = false;  // a split that gave up writes NaN pairs
#pragma unroll
  for (int sp = 0; sp < kMaxSplits; ++sp)
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      m_s[sp][x] = -INFINITY;
      l_s[sp][x] = 0.0f;
      if (sp < S) {
        const float* ml = p.part_ml + ((cta0 + sp) * 3 + x) * 2 * kRows;
        m_s[sp][x] = ml[row];
        l_s[sp][x] = ml[kRows + row];
        aborted |= isnan(m_s[sp][x]) || isnan(l_s[sp][x]);
      }
    }
  float w[kMaxSplits][3], inv[3];
#pragma unroll
  for (int x = 0; x < 3; ++x) {
    float mx = -INFINITY;
#pragma unroll
    for (int sp = 0; sp < kMaxSplits; ++sp) mx = fmaxf(mx, m_s[sp][x]);
    float L = 0.0f;
#pragma unroll
    for (int sp = 0; sp < kMaxSplits; ++sp) {
      w[sp][x] = m_s[sp][x] == -INFINITY ? 0.0f : exp2f(m_s[sp][x] - mx);
      L = fmaf(w[sp][x], l_s[sp][x], L);
    }
    inv[x] = L > 0.0f ? 1.0f / L : 0.0f;
  }
  float err[2] = {0.0f, 0.0f};
  if (valid && !aborted) {
    for (int c = quarter * (D / kCombineQuarters); c < (quarter + 1) * (D / kCombineQuarters);
         ++c) {
      float o[3] = {0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int sp = 0; sp < kMaxSplits; ++sp) {
        if (sp >= S) break;
#pragma unroll
        for (int x = 0; x < 3; ++x)
          o[x] = fmaf(w[sp][x], __ldg(p.part_o + (((cta0 + sp) * 3 + x) * D + c) * kRows + row),
                      o[x]);
      }
      const float oF = o[0] * inv[0];
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const float dlt = o[1 + x] * inv[1 + x] - oF;
        err[x] = fmaf(dlt, dlt, err[x]);
      }
    }
  }
  red[0][quarter][row] = aborted ? __int_as_float(0x7fc00000) : err[0];
  red[1][quarter][row] = aborted ? __int_as_float(0x7fc00000) : err[1];
  __syncthreads();
  if (threadIdx.x < 2) {
    const int x = threadIdx.x;
    float acc = 0.0f;
    for (int i = 0; i < kRows; ++i)
      for (int q = 0; q < kCombineQuarters; ++q) acc += red[x][q][i];
    p.partial[(static_cast<size_t>(bh) * 2 + x) * p.n_tiles + tile] = acc;
  }
}

// Sums the per-tile partial errors of each head in tile order and labels it.
__global__ void profile_finalize_kernel(const float* __restrict__ partial, int32_t BH,
                                        int32_t n_tiles, float inv_count,
                                        int8_t* __restrict__ labels, float* __restrict__ mse) {
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= BH) return;
  float e[2];
  for (int x = 0; x < 2; ++x) {
    const float* src = partial + (static_cast<size_t>(bh) * 2 + x) * n_tiles;
    float acc = 0.0f;
    for (int t = 0; t < n_tiles; ++t) acc += src[t];
    e[x] = acc * inv_count;
  }
  labels[bh] = e[1] < e[0] ? SVG_HEAD_TEMPORAL : SVG_HEAD_SPATIAL;
  if (mse != nullptr) {
    mse[2 * bh] = e[0];
    mse[2 * bh + 1] = e[1];
  }
}

template <int D>
cudaError_t launch_impl(const Dims& d, const ProfParams& pp, int8_t* labels, float* mse,
                        cudaStream_t stream) {
  using C = PCfg<D>;
  auto kern = profile_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(pp.n_tiles, d.BH, pp.n_splits), kThreads, C::kSmem, stream>>>(pp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (pp.n_splits > 1) {
    profile_combine_kernel<D>
        <<<dim3(pp.n_tiles, d.BH), kRows * kCombineQuarters, 0, stream>>>(pp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const float inv = 1.0f / (static_cast<float>(pp.n_samples) * static_cast<float>(D));
  profile_finalize_kernel<<<(d.BH + 127) / 128, 128, 0, stream>>>(pp.partial, d.BH, pp.n_tiles,
                                                                  inv, labels, mse);
  return cudaGetLastError();
}

}  // namespace

int32_t profile_tiles(int32_t n_samples) { return (n_samples + kRows - 1) / kRows; }

// Key-range splits per (head, sample tile): the count in 1..4 (never more than
// the key tiles) that fills the last wave best on a B200's 148 SMs, one CTA
// each; ties go to fewer splits.
int32_t profile_splits(const Dims& d, int32_t n_samples) {
  constexpr int64_t kSMs = 148;
  const int64_t ctas = static_cast<int64_t>(d.BH) * profile_tiles(n_samples);
  const int32_t nkt = (d.N + kKeys - 1) / kKeys;
  int32_t best = 1;
  double best_fill = 0.0;
  for (int32_t sp = 1; sp <= kMaxSplits && sp <= nkt; ++sp) {
    const int64_t c = ctas * sp;
    const double fill = static_cast<double>(c) / static_cast<double>((c + kSMs - 1) / kSMs * kSMs);
    if (fill > best_fill + 1e-9) {
      best = sp;
      best_fill = fill;
    }
  }
  return best;
}

size_t profile_workspace_bytes(const Dims& d, int32_t n_samples, int32_t n_splits) {
  const size_t ctas = static_cast<size_t>(d.BH) * profile_tiles(n_samples);
  size_t bytes = ctas * 2 * sizeof(float);  // per-tile errors
  if (n_splits > 1) {
    bytes = (bytes + 255) / 256 * 256;
    bytes += ctas * n_splits * 3 * static_cast<size_t>(d.d) * kRows * sizeof(float);
    bytes += ctas * n_splits * 3 * 2 * kRows * sizeof(float);
  }
  return bytes;
}

// ---------------------------------------------------------------------------
// Fixed scratch for svg_profile_heads_noalloc: the per-tile partial sums live
// in this module's own device array instead of caller memory. Every GPU that
// loads the library keeps one copy until the process exits. The profiling
// kernel writes every slot it later reads, so nothing needs clearing between
// calls; calls that overlap on the GPU share it and race.
namespace {
constexpr size_t kNoAllocScratchBytes = 256 * 1024;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mutex;
float* g_scratch_ptr[kMaxScratchDevices] = {};
void* g_scratch_ctx[kMaxScratchDevices] = {};  // context the cached address belongs to

// Device address of the current device's copy of g_noalloc_scratch. In host
// code the array's name is only a stand-in, so the address is looked up with
// cudaGetSymbolAddress with that device current: on the first call on each
// device, and again whenever the device's context changed since (after a
// cudaDeviceReset the module is loaded again, at another address).
cudaError_t noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
  // No lock is held while the runtime or the driver is called.
  void* ctx = current_context();
  {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] != nullptr && ctx != nullptr && g_scratch_ctx[dev] == ctx) {
      *out = g_scratch_ptr[dev];
      return cudaSuccess;
    }
  }
  void* ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);  // initialises the context if needed
  if (e != cudaSuccess) return e;
  void* now = current_context();
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  g_scratch_ptr[dev] = static_cast<float*>(ptr);
  g_scratch_ctx[dev] = now;
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}
}  // namespace

size_t profile_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

cudaError_t launch_profile_noalloc(const Dims& d, const ProfileArgs& a, int* status,
                                   cudaStream_t stream) {
  float* scratch = nullptr;
  const cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  ProfileArgs args = a;
  args.partial = scratch;
  args.n_splits = 1;
  return launch_profile(d, args, status, stream);
}

cudaError_t launch_profile(const Dims& d, const ProfileArgs& a, int* status, cudaStream_t stream) {
  ProfParams pp;
  memset(&pp, 0, sizeof(pp));
  if (!make_tmap_bf16(&pp.tm_k, a.k, d.d, d.N, d.BH, kKeys) ||
      !make_tmap_bf16(&pp.tm_v, a.v, d.d, d.N, d.BH, kKeys))
    return cudaErrorInvalidValue;
  pp.q = a.q;
  pp.sample_idx = a.sample_idx;
  pp.partial = a.partial;
  pp.n_splits = a.n_splits;
  if (a.n_splits > 1) {
    const size_t ctas = static_cast<size_t>(d.BH) * profile_tiles(a.n_samples);
    uint8_t* base = reinterpret_cast<uint8_t*>(a.partial);
    const size_t off_o = (ctas * 2 * sizeof(float) + 255) / 256 * 256;
    pp.part_o = reinterpret_cast<float*>(base + off_o);
    pp.part_ml = pp.part_o + ctas * a.n_splits * 3 * static_cast<size_t>(d.d) * kRows;
  }
  pp.status = status;
  pp.n_samples = a.n_samples;
  pp.n_tiles = profile_tiles(a.n_samples);
  pp.N = d.N;
  pp.Nv = d.Nv;
  pp.T = d.T;
  pp.P = d.P;
  pp.s = d.s;
  pp.w = d.w;
  pp.nkt = (d.N + kKeys - 1) / kKeys;
  pp.scale_log2 = d.scale * 1.4426950408889634f;
  if (d.d == 128) return launch_impl<128>(d, pp, a.labels, a.mse, stream);
  return launch_impl<64>(d, pp, a.labels, a.mse, stream);
}

}  // namespace svg
