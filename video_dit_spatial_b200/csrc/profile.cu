// Online profiling of Sparse VideoGen (arXiv 2502.01776 abstract: "an online
// profiling strategy to capture the dynamic sparse patterns and predict the
// type of attention head"). For sampled query rows of every head, full
// attention is compared with spatial-masked and temporal-masked attention by
// the mean squared error of the outputs; the mask with the smaller error names
// the head's type.
//
// One CTA = one (b*H + h, mask X in {spatial, temporal}, tile of 128 sampled
// rows). It runs flash attention of its 128 gathered query rows over ALL keys
// (128-key tiles, TMA-fed), keeping two online softmaxes side by side: the
// full one and the token-level masked one, each with its own running maximum.
//
// 320 threads: warps 0-7 softmax, warp 8 TMA producer, warp 9 MMA issuer.
// Warps w and w+4 own the same 32 query rows (TMEM lanes 32*(w%4)..+31) and
// split each 128-key tile into columns [0,64) and [64,128); they exchange row
// maxima through shared memory (one 64-thread named barrier per warp pair)
// and keep partial row sums that are added once at the end.
// Tensor memory: S double buffer (columns 0 and 128), O_full (256), O_X
// (256 + d); P_full and P_X (bf16) overwrite the two halves of their S buffer.
// The allowed keys of a row inside a tile are at most a few index runs
// (spatial: the frames [f-s, f+s]; temporal: positions [p-w, p+w] of each
// frame; text keys always), built as bit ranges. P_X = P_full * 2^(mF - mX) on
// allowed keys; the masked product P_X V is skipped for key tiles where no row
// of the CTA has an allowed key. Each CTA reduces sum((O_X - O_full)^2) over
// its rows in a fixed order into the workspace; a second kernel adds the
// tiles in a fixed order and labels the head.
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace svg {
namespace {

constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = (kSoftmaxWarps + 2) * 32;
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;
constexpr int kTile = 128;  // sampled rows per CTA and keys per tile
constexpr int kHalf = 64;   // keys per softmax thread per tile
constexpr float kRebaseLog2 = 8.0f;

struct PBarriers {
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[2], p_full[2];
  uint64_t o_full, o_final, drain;
  uint32_t tmem_base;
  int abort_flag;
  int x_active[2][kSoftmaxWarps];
  float xmax[2][2][128];  // [half][full, masked][row]
  float xsum[2][2][128];  // [half][full, masked][row]
  float red[2][128];
  int pair_fail[4][2];
};

template <int D>
struct PCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPanel = 128 * 128;  // 128 rows x 128 B
  static constexpr int kQBytes = kPanels * kPanel;
  static constexpr int kKVBytes = kPanels * kPanel;
  // K is released right after its QK product, V only after its PV products,
  // so K gets the deeper ring.
  static constexpr int kKStages = 3;
  static constexpr int kVStages = D == 128 ? 2 : 3;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kVStages * kKVBytes;
  static constexpr int kBarBytes = (static_cast<int>(sizeof(PBarriers)) + 127) / 128 * 128;
  static constexpr int kUsed = kOffBar + kBarBytes + 1024;
  static constexpr int kSmem = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColOF = 256, kColOX = 256 + D;
  static_assert(kOffBar + kBarBytes + 1024 <= kSmem, "bookkeeping must fit the allocation");
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
};

struct __align__(64) ProfParams {
  CUtensorMap tm_k, tm_v;
  const svg_bf16* q;
  const int32_t* sample_idx;
  float* partial;  // [BH][2][n_tiles]
  int* status;
  int32_t n_samples, n_tiles;
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1) profile_kernel(const __grid_constant__ ProfParams p) {
  using C = PCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  PBarriers* bar = reinterpret_cast<PBarriers*>(smem + C::kOffBar);
  volatile int* abort_flag = &bar->abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  // Launch order: every temporal-mask CTA (the slower kind: its allowed keys
  // reach every frame) before any spatial-mask CTA, heads in order.
  const int tile = blockIdx.x;
  const int bh = blockIdx.y;
  const int X = 1 - static_cast<int>(blockIdx.z);  // 0: spatial mask, 1: temporal mask
  const int n = p.nkt;

  if (warp == 0) {
    tmem_alloc(&bar->tmem_base, C::kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 32) {
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
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
    const int si = tile * kTile + row;
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
      *reinterpret_cast<uint4*>(sQ + pn * C::kPanel + row * 128 + ((ci ^ (row & 7)) << 4)) = v;
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
          const int st = j % C::kKStages;
          ok = mbar_wait(&bar->k_empty[st], ((j / C::kKStages) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          mbar_arrive_expect_tx(&bar->k_full[st], C::kKVBytes);
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d_hint(sK + st * C::kKVBytes + pn * C::kPanel, &p.tm_k, &bar->k_full[st],
                             pn * 64, j * kTile, bh, keep);
          k_issued = j + 1;
        }
        if (j >= 1) {
          const int jv = j - 1;
          const int st = jv % C::kVStages;
          ok = mbar_wait(&bar->v_empty[st], ((jv / C::kVStages) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          mbar_arrive_expect_tx(&bar->v_full[st], C::kKVBytes);
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d_hint(sV + st * C::kKVBytes + pn * C::kPanel, &p.tm_v, &bar->v_full[st],
                             pn * 64, jv * kTile, bh, keep);
          v_issued = jv + 1;
        }
      }
      if (*abort_flag) {
        // Let every copy this thread started land before the CTA retires.
        for (int j = (k_issued > C::kKStages ? k_issued - C::kKStages : 0); j < k_issued; ++j) {
          long long t0 = clock64();
          while (!mbar_try_wait(&bar->k_full[j % C::kKStages], (j / C::kKStages) & 1) &&
                 clock64() - t0 < kWaitLimitCycles) {
          }
        }
        for (int j = (v_issued > C::kVStages ? v_issued - C::kVStages : 0); j < v_issued; ++j) {
          long long t0 = clock64();
          while (!mbar_try_wait(&bar->v_full[j % C::kVStages], (j / C::kVStages) & 1) &&
                 clock64() - t0 < kWaitLimitCycles) {
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane_id() == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kTile, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      bool x_started = false;
      for (int j = 0; j <= n; ++j) {
        if (j < n) {
          const int st = j % C::kKStages;
          const uint32_t s_col = tmem + ((j & 1) ? C::kColS1 : C::kColS0);
          if (!mbar_wait(&bar->k_full[st], (j / C::kKStages) & 1, abort_flag, p.status)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kPanel + (kk & 3) * 32;
            mma_bf16_ss(s_col, sdesc_sw128(q_addr + off, 16, 1024),
                        sdesc_sw128(k_addr + st * C::kKVBytes + off, 16, 1024), idesc_qk,
                        kk > 0 ? 1u : 0u);
          }
          tc_commit(&bar->s_full[j & 1]);
          tc_commit(&bar->k_empty[st]);  // K(j) is free once QK_j retires
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj % C::kVStages;
          const int sb = jj & 1;
          const uint32_t p_col = tmem + (sb ? C::kColS1 : C::kColS0);
          if (!mbar_wait(&bar->p_full[sb], (jj >> 1) & 1, abort_flag, p.status)) break;
          if (!mbar_wait(&bar->v_full[st], (jj / C::kVStages) & 1, abort_flag, p.status)) break;
          tc_fence_after();
          const volatile int* xa = bar->x_active[sb];
          int x_any = 0;
#pragma unroll
          for (int w = 0; w < kSoftmaxWarps; ++w) x_any |= xa[w];
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint64_t b = sdesc_sw128(v_addr + st * C::kKVBytes + kk * 16 * 128, C::kPanel,
                                           1024);
            mma_bf16_ts(tmem + C::kColOF, p_col + kk * 8, b, idesc_pv,
                        (jj > 0 || kk > 0) ? 1u : 0u);
          }
          if (x_any) {
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t b = sdesc_sw128(v_addr + st * C::kKVBytes + kk * 16 * 128,
                                             C::kPanel, 1024);
              mma_bf16_ts(tmem + C::kColOX, p_col + 64 + kk * 8, b, idesc_pv,
                          (x_started || kk > 0) ? 1u : 0u);
            }
            x_started = true;
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
    const int group = warp & 3;  // rows 32*group .. +31 (TMEM lane quarter)
    const int c_base = half * kHalf;  // this thread's key columns within a tile
    const bool row_valid = qrow >= 0;
    const int qi = row_valid ? qrow : 0;
    const int f_i = qi / p.P;
    const int p_i = qi - f_i * p.P;
    // Allowed video keys of this row: spatial = the frames [f_i - s, f_i + s]
    // (one index run); temporal = positions [p_i - w, p_i + w] of every frame
    // (one run per frame). Text keys [Nv, N) are allowed by both.
    const int s_lo = max(f_i - p.s, 0) * p.P;  // frames [f_i - s, f_i + s] as one index run
    const int s_hi = static_cast<int>(min(static_cast<long long>(f_i) + p.s + 1,
                                          static_cast<long long>(p.T))) * p.P;
    const int t_lo = max(p_i - p.w, 0);
    const int t_hi = static_cast<int>(
        min(static_cast<long long>(p_i) + p.w, static_cast<long long>(p.P - 1)));
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(group * 32) << 16);
    float mF = -INFINITY, lF = 0.0f, mX = -INFINITY, lX = 0.0f;
    bool ok = true;
    int fs0 = 0;  // start of the frame holding this thread's first key of the tile
    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      const uint32_t s_col = lane_base + (sb ? C::kColS1 : C::kColS0);
      const int k0 = j * kTile + c_base;       // first key of this thread's half
      const int kvalid = max(0, min(kHalf, p.N - k0));
      const int k_end = k0 + kvalid;           // exclusive
      uint32_t bits[2] = {0u, 0u};  // allowed keys k0 + [0, 64) of this row
      if (row_valid && kvalid > 0) {
        if (k_end > p.Nv) set_bit_range64(bits, max(p.Nv, k0) - k0, kvalid);
        if (k0 < p.Nv) {
          const int v_end = min(k_end, p.Nv);
          if (X == 0) {
            set_bit_range64(bits, max(s_lo, k0) - k0, min(s_hi, v_end) - k0);
          } else {
            // frames overlapping the half tile (at most two when P >= 64);
            // fs0 tracks the start of the frame holding k0 across tiles
            while (fs0 + p.P <= k0) fs0 += p.P;
            for (int fs = fs0; fs < v_end; fs += p.P)
              set_bit_range64(bits, max(fs + t_lo, k0) - k0, min(fs + t_hi + 1, v_end) - k0);
          }
        }
      }
      const bool any_x = (bits[0] | bits[1]) != 0u;
      const int warp_any = __any_sync(0xffffffffu, any_x) ? 1 : 0;

      if (ok && !mbar_wait(&bar->s_full[sb], (j >> 1) & 1, abort_flag, p.status)) ok = false;
      // Both warps of a pair must take the same path through pair_sync (an
      // unbounded barrier), so they agree on leaving the loop through it.
      if (__any_sync(0xffffffffu, !ok)) ok = false;
      if (lane_id() == 0) bar->pair_fail[group][half] = ok ? 0 : 1;
      float a0 = -INFINITY, a1 = -INFINITY, b0 = -INFINITY, b1 = -INFINITY;
      uint32_t sr[kHalf];
      if (ok) {
        tc_fence_after();
        tmem_ld_32x32b_x32(s_col + c_base, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld_32x32b_x32(s_col + c_base + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
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
        // The masked maximum of this half can only move the masked base when
        // the half's full maximum exceeds mX + 2^8; otherwise report -inf: the
        // combined decision and the new base are unchanged.
        const bool need_m = any_x && fmaxf(a0, a1) * p.scale_log2 > mX + kRebaseLog2;
        if (__any_sync(0xffffffffu, need_m)) {
#pragma unroll
          for (int c = 0; c < kHalf; c += 4) {
            const float x0 = ((bits[c >> 5] >> (c & 31)) & 1u) ? u2f(sr[c]) : -INFINITY;
            const float x1 = ((bits[(c + 1) >> 5] >> ((c + 1) & 31)) & 1u) ? u2f(sr[c + 1]) : -INFINITY;
            const float x2 = ((bits[(c + 2) >> 5] >> ((c + 2) & 31)) & 1u) ? u2f(sr[c + 2]) : -INFINITY;
            const float x3 = ((bits[(c + 3) >> 5] >> ((c + 3) & 31)) & 1u) ? u2f(sr[c + 3]) : -INFINITY;
            b0 = fmax3(b0, x0, x1);
            b1 = fmax3(b1, x2, x3);
          }
        }
      }
      // exchange the half-row maxima with the partner warp
      bar->xmax[half][0][row] = fmaxf(a0, a1);
      bar->xmax[half][1][row] = fmaxf(b0, b1);
      pair_sync(group);
      const float tF = fmaxf(bar->xmax[0][0][row], bar->xmax[1][0][row]) * p.scale_log2;
      const float tX = fmaxf(bar->xmax[0][1][row], bar->xmax[1][1][row]) * p.scale_log2;
      const int pair_failed = bar->pair_fail[group][0] | bar->pair_fail[group][1];
      pair_sync(group);  // the exchange slots are rewritten next tile
      if (pair_failed) {
        ok = false;
        break;
      }

      const bool rbF = tF > mF + kRebaseLog2;
      const bool rbX = tX > mX + kRebaseLog2;
      const float mF_new = rbF ? tF : mF, mX_new = rbX ? tX : mX;
      const float aF = rbF ? fast_exp2(mF - mF_new) : 1.0f;
      const float aX = rbX ? fast_exp2(mX - mX_new) : 1.0f;
      const float uF = mF_new == -INFINITY ? 0.0f : mF_new;
      const float uX = mX_new == -INFINITY ? 0.0f : mX_new;
      // P_X = P_full * 2^(mF - mX) on allowed keys, unless the masked base is
      // so far below the full one that 2^(x - mF) could flush to zero; those
      // (rare) warps evaluate the masked exponentials directly.
      // (With no allowed key seen yet, mX is -inf and every P_X is zero.)
      const float gap = uF - uX;
      const bool direct = mX_new != -INFINITY && gap > 64.0f;
      const float kX = direct ? 0.0f : fast_exp2(gap);
      const bool warp_direct = __any_sync(0xffffffffu, direct);
      // Warp-uniform shapes of the allowed-key set of this half tile.
      const bool w_none = __all_sync(0xffffffffu, (bits[0] | bits[1]) == 0u);
      const bool w_all = __all_sync(0xffffffffu, (bits[0] & bits[1]) == 0xffffffffu);
      const int shape = warp_direct ? 3 : (w_none ? 1 : (w_all ? 2 : 0));
      float sF0 = 0.0f, sF1 = 0.0f, sX0 = 0.0f, sX1 = 0.0f;
#pragma unroll
      for (int ch = 0; ch < kHalf / 32; ++ch) {
        uint32_t pkF[16], pkX[16];
        if (shape == 1) {  // no allowed key in this half for the whole warp
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c0 = ch * 32 + 2 * i;
            float y0, y1;
            ffma2(y0, y1, u2f(sr[c0]), u2f(sr[c0 + 1]), p.scale_log2, p.scale_log2, -uF, -uF);
            const float f0 = fast_exp2(y0), f1 = fast_exp2(y1);
            fadd2(sF0, sF1, sF0, sF1, f0, f1);
            pkF[i] = pack_bf16x2(f0, f1);
            pkX[i] = 0u;
          }
        } else if (shape == 2) {  // every key allowed for the whole warp
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c0 = ch * 32 + 2 * i;
            float y0, y1, g0, g1;
            ffma2(y0, y1, u2f(sr[c0]), u2f(sr[c0 + 1]), p.scale_log2, p.scale_log2, -uF, -uF);
            const float f0 = fast_exp2(y0), f1 = fast_exp2(y1);
            ffma2(g0, g1, f0, f1, kX, kX, 0.0f, 0.0f);
            fadd2(sF0, sF1, sF0, sF1, f0, f1);
            fadd2(sX0, sX1, sX0, sX1, g0, g1);
            pkF[i] = pack_bf16x2(f0, f1);
            pkX[i] = pack_bf16x2(g0, g1);
          }
        } else if (shape == 0) {  // general: per-key selection
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c0 = ch * 32 + 2 * i;
            float y0, y1;
            ffma2(y0, y1, u2f(sr[c0]), u2f(sr[c0 + 1]), p.scale_log2, p.scale_log2, -uF, -uF);
            const float f0 = fast_exp2(y0), f1 = fast_exp2(y1);
            const float g0 = ((bits[ch] >> (2 * i)) & 1u) ? f0 * kX : 0.0f;
            const float g1 = ((bits[ch] >> (2 * i + 1)) & 1u) ? f1 * kX : 0.0f;
            fadd2(sF0, sF1, sF0, sF1, f0, f1);
            fadd2(sX0, sX1, sX0, sX1, g0, g1);
            pkF[i] = pack_bf16x2(f0, f1);
            pkX[i] = pack_bf16x2(g0, g1);
          }
        } else {  // some row's masked base is far below its full base
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c0 = ch * 32 + 2 * i;
            float y0, y1;
            ffma2(y0, y1, u2f(sr[c0]), u2f(sr[c0 + 1]), p.scale_log2, p.scale_log2, -uF, -uF);
            const float f0 = fast_exp2(y0), f1 = fast_exp2(y1);
            const bool in0 = (bits[ch] >> (2 * i)) & 1u;
            const bool in1 = (bits[ch] >> (2 * i + 1)) & 1u;
            float g0 = in0 ? f0 * kX : 0.0f;
            float g1 = in1 ? f1 * kX : 0.0f;
            if (direct) {
              g0 = in0 ? fast_exp2(fmaf(u2f(sr[c0]), p.scale_log2, -uX)) : 0.0f;
              g1 = in1 ? fast_exp2(fmaf(u2f(sr[c0 + 1]), p.scale_log2, -uX)) : 0.0f;
            }
            fadd2(sF0, sF1, sF0, sF1, f0, f1);
            fadd2(sX0, sX1, sX0, sX1, g0, g1);
            pkF[i] = pack_bf16x2(f0, f1);
            pkX[i] = pack_bf16x2(g0, g1);
          }
        }
        // keys k -> column k/2: this half's 64 keys fill 32 columns
        tmem_st_32x32b_x16(s_col + half * 32 + ch * 16, pkF);
        tmem_st_32x32b_x16(s_col + 64 + half * 32 + ch * 16, pkX);
      }
      lF = lF * aF + (sF0 + sF1);
      lX = lX * aX + (sX0 + sX1);
      mF = mF_new;
      mX = mX_new;
      tmem_st_wait();
      if (lane_id() == 0) bar->x_active[sb][warp] = warp_any;

      // Re-base this half's columns of O_full / O_X once PV_{j-1} has landed.
      const bool wF = __any_sync(0xffffffffu, rbF);
      const bool wX = __any_sync(0xffffffffu, rbX);
      if (j > 0 && (wF || wX)) {
        // A failed wait is reported through the pair exchange of the next tile.
        if (!mbar_wait(&bar->o_full, (j - 1) & 1, abort_flag, p.status)) ok = false;
        tc_fence_after();
#pragma unroll
        for (int which = 0; which < 2 && ok; ++which) {
          if (which == 0 ? !wF : !wX) continue;
          const float a = which == 0 ? aF : aX;
          const uint32_t ocol = lane_base + (which == 0 ? C::kColOF : C::kColOX) + half * (D / 2);
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(ocol + ch * 32, o);
            tmem_ld_wait();
            reg_fence(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(u2f(o[i]) * a);
            tmem_st_32x32b_x32(ocol + ch * 32, o);
          }
        }
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&bar->p_full[sb]);
    }

    // ---- per-row squared error over this half's d/2 channels
    bar->xsum[half][0][row] = lF;
    bar->xsum[half][1][row] = lX;
    if (ok && n > 0) ok = mbar_wait(&bar->o_final, 0, abort_flag, p.status);
    softmax_sync();
    const float LF = bar->xsum[0][0][row] + bar->xsum[1][0][row];
    const float LX = bar->xsum[0][1][row] + bar->xsum[1][1][row];
    tc_fence_after();
    float err = 0.0f;
    const bool all_ok = __all_sync(0xffffffffu, ok);
    if (all_ok && n > 0) {
      const float iF = LF > 0.0f ? 1.0f / LF : 0.0f;
      const float iX = LX > 0.0f ? 1.0f / LX : 0.0f;
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch) {
        uint32_t oF[32], oX[32];
        tmem_ld_32x32b_x32(lane_base + C::kColOF + half * (D / 2) + ch * 32, oF);
        tmem_ld_32x32b_x32(lane_base + C::kColOX + half * (D / 2) + ch * 32, oX);
        tmem_ld_wait();
        reg_fence(oF);
        reg_fence(oX);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float dlt = u2f(oX[i]) * iX - u2f(oF[i]) * iF;
          err = fmaf(dlt, dlt, err);
        }
      }
    }
    bar->red[half][row] = row_valid ? err : 0.0f;
    if (!all_ok) atomicOr(&bar->abort_flag, 1);
    softmax_sync();
    if (tid == 0) {
      float acc = 0.0f;
      for (int i = 0; i < 128; ++i) acc += bar->red[0][i] + bar->red[1][i];
      p.partial[(static_cast<size_t>(bh) * 2 + X) * p.n_tiles + tile] =
          *abort_flag ? __int_as_float(0x7fc00000) : acc;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
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
  kern<<<dim3(pp.n_tiles, d.BH, 2), kThreads, C::kSmem, stream>>>(pp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const float inv = 1.0f / (static_cast<float>(pp.n_samples) * static_cast<float>(D));
  profile_finalize_kernel<<<(d.BH + 127) / 128, 128, 0, stream>>>(pp.partial, d.BH, pp.n_tiles,
                                                                  inv, labels, mse);
  return cudaGetLastError();
}

}  // namespace

int32_t profile_tiles(int32_t n_samples) { return (n_samples + kTile - 1) / kTile; }

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

// Device address of the current device's copy of g_noalloc_scratch. In host
// code the array's name is only a stand-in, so the address is looked up with
// cudaGetSymbolAddress, once per device, with that device current.
cudaError_t noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(ptr);
  }
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
  return launch_profile(d, args, status, stream);
}

cudaError_t launch_profile(const Dims& d, const ProfileArgs& a, int* status, cudaStream_t stream) {
  ProfParams pp;
  memset(&pp, 0, sizeof(pp));
  if (!make_tmap_bf16(&pp.tm_k, a.k, d.d, d.N, d.BH, kTile) ||
      !make_tmap_bf16(&pp.tm_v, a.v, d.d, d.N, d.BH, kTile))
    return cudaErrorInvalidValue;
  pp.q = a.q;
  pp.sample_idx = a.sample_idx;
  pp.partial = a.partial;
  pp.status = status;
  pp.n_samples = a.n_samples;
  pp.n_tiles = profile_tiles(a.n_samples);
  pp.N = d.N;
  pp.Nv = d.Nv;
  pp.T = d.T;
  pp.P = d.P;
  pp.s = d.s;
  pp.w = d.w;
  pp.nkt = (d.N + kTile - 1) / kTile;
  pp.scale_log2 = d.scale * 1.4426950408889634f;
  if (d.d == 128) return launch_impl<128>(d, pp, a.labels, a.mse, stream);
  return launch_impl<64>(d, pp, a.labels, a.mse, stream);
}

}  // namespace svg
